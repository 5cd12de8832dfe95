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
// operand of QK^T, V transposed for the A operand of PV).  The ring is split
// into one sub-ring per consumer warp (stages w, w + NW, w + 2 NW, ... belong
// to warp w), and chunk j of every work item goes to warp j mod NW: a warp
// consumes the fills of its own stages in order, so it never waits on a
// barrier phase that a slower warp has not reached yet (parity waits cannot
// tell phase k from phase k+2), and which warp sums which chunk -- the fp32
// summation order -- does not depend on how items are handed out, so results
// are reproducible run to run.
// The consumer warps (two: small CTAs, more of them per SM, measured best),
// each with its own online softmax, merge through shared
// memory.  Rows past the context are masked out of the scores, and the
// matching V rows are zeroed in shared memory before PV (0 * NaN would poison
// the sum).
//
// Two schedules share this code:
//  * mma_decode_kernel: one CTA per (sequence, kv head, partition);
//  * mma_decode_persistent_kernel (up to 1024 sequences, split or not): a few
//    CTAs per SM take work items
//    (sequence, kv head, partition) from a ticket counter -- every full
//    partition first, then the partial last partitions longest first -- and
//    the producer
//    streams chunks across item boundaries without draining the ring.  The
//    items' query tiles travel through a small queue (bulk copies) with their
//    descriptors, and each finished item is merged while the next streams in.
//    (Merging the split-K partitions inside this kernel, by the CTA that
//    stores a context's last partition, was measured slower than the separate
//    merge kernel: those merges land at the end of the launch.)
#include "common.cuh"
#include "kernels.h"

#include <atomic>

namespace pkv {
namespace {

constexpr int NW = MMA_CONSUMER_WARPS;
constexpr int CHUNK = 16;  // tokens per ring stage
constexpr int IQ = 1;      // item-queue depth of the persistent kernel (a deeper queue costs occupancy)

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
// of token row `tok` in a stage tile laid out as [D/64 slices][16 rows][128 B]
// with the 128-byte swizzle (unit index XOR row mod 8).
__device__ __forceinline__ uint32_t swz_addr(uint32_t tile, int tok, int colh) {
  const int sl = colh >> 6;
  const int unit = (colh & 63) >> 3;
  return tile + sl * (CHUNK * 128) + tok * 128 + ((unit ^ (tok & 7)) << 4);
}

template <int D>
struct StageGeom {
  static constexpr int NSL = D / 64;                           // 64-column slices
  static constexpr uint32_t SLICE_BYTES = CHUNK * 128;
  static constexpr uint32_t TILE_BYTES = NSL * SLICE_BYTES;    // K (or V) of one stage
  static constexpr int MT = D / 16;                            // 16-wide slices of D
  static constexpr int OSTRIDE = D + 4;                        // padded merge rows
  // one consumer warp's softmax state for the per-item merge: max[8], sum[8], o[8][OSTRIDE]
  static constexpr int STATE_FLOATS = 16 + 8 * OSTRIDE;
  static_assert(STATE_FLOATS * 4 <= 2 * TILE_BYTES, "a warp's state must fit one ring stage");
};

// ---- producer side ---------------------------------------------------------------

// Issues the TMA copies of chunk c (16 tokens) of an item whose table window
// (entries w0 .. w0+31 of the item's blocks) is staged in s_ids.
template <int D, int BS>
__device__ __forceinline__ void issue_stage(uint32_t kdst, uint32_t full, const int* s_ids, int w0,
                                            int c, int nblk, int kvh, int num_kv_heads,
                                            const CUtensorMap* km, const CUtensorMap* vm,
                                            uint64_t policy) {
  using Geo = StageGeom<D>;
  constexpr int CB = BS < CHUNK ? BS : CHUNK;  // rows per TMA box
  constexpr int NB = CHUNK / CB;               // boxes per stage and slice
  constexpr uint32_t BOX_BYTES = CB * 128;
  const uint32_t vdst = kdst + Geo::TILE_BYTES;
  const int first = c * NB;  // first block of the stage (bs 8)
  const int nb = BS >= CHUNK ? 1 : min(NB, nblk - first);
  mbar_arrive_expect_tx(full, 2u * nb * Geo::NSL * BOX_BYTES);
  for (int k = 0; k < nb; ++k) {
    int y;
    if (BS >= CHUNK) {
      const int tok = c * CHUNK;
      y = (s_ids[tok / BS - w0] * num_kv_heads + kvh) * BS + tok % BS;
    } else {
      y = (s_ids[first + k - w0] * num_kv_heads + kvh) * BS;
    }
#pragma unroll
    for (int sl = 0; sl < Geo::NSL; ++sl) {
      const uint32_t off = sl * Geo::SLICE_BYTES + k * BOX_BYTES;
      tensor_load_2d(kdst + off, km, sl * 64, y, full, policy);
      tensor_load_2d(vdst + off, vm, sl * 64, y, full, policy);
    }
  }
}

// Fill counts of the consumer warps' sub-rings: stage (k mod SPW) * NW + w
// takes warp w's k-th fill, SPW = stages / NW.
struct RingFills {
  int n[NW];
  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int w = 0; w < NW; ++w) n[w] = 0;
  }
  // after an item of nchunks chunks (chunk j went to warp j mod NW)
  __device__ __forceinline__ void advance(int nchunks) {
#pragma unroll
    for (int w = 0; w < NW; ++w) n[w] += (nchunks - w + NW - 1) / NW;
  }
};

__device__ __forceinline__ int ring_stage(int k, int warp, int spw) { return (k % spw) * NW + warp; }

// Streams the nchunks chunks of one item (its table row starts at `row`) into
// the ring: chunk c goes to warp c mod NW's sub-ring, as that warp's fill
// base.n[w] + c / NW.  Run by the whole producer warp; lane 0 issues.  With a
// fused append (new_tok >= 0: the item ends its context, and its token new_tok
// is the new one) the warp writes the new K/V rows of sequence b, kv head kvh,
// into their slot before it issues the chunk that reads them.  Returns false
// (warp-uniform) when it gave up; lane 0's issued.n[w] counts the fills issued
// to warp w so far.
template <int D, int BS>
__device__ bool produce_item(const int32_t* row, int nblk, int nchunks, const RingFills& base,
                             int kvh, int b, int new_tok, const DecodeParams& p, int* s_ids,
                             uint64_t* bars, int stages, uint32_t ring, const CUtensorMap* km,
                             const CUtensorMap* vm, uint64_t policy, volatile int* abort_flag,
                             int lane, RingFills& issued) {
  using Geo = StageGeom<D>;
  NewRows<D, 1> fresh;
  if (new_tok >= 0) fresh.load(p.k_new, p.v_new, b, p.num_kv_heads, kvh, lane);
  const int spw = stages / NW;
  // issues chunk c (lane 0 only); false when the wait for a free stage gave up
  auto issue = [&](int c, int w0) -> bool {
    const int w = c % NW;
    const int k = base.n[w] + c / NW;
    const int st = ring_stage(k, w, spw);
    const int round = k / spw;
    if (round > 0 && !mbar_wait(smem_u32(&bars[stages + st]), (round - 1) & 1)) {
      *abort_flag = 1;
      flag_error(p.err, ERR_TIMEOUT);
      return false;
    }
    issue_stage<D, BS>(ring + (uint32_t)st * 2 * Geo::TILE_BYTES, smem_u32(&bars[st]), s_ids, w0,
                       c, nblk, kvh, p.num_kv_heads, km, vm, policy);
    issued.n[w] = k + 1;
    return true;
  };
  bool ok = true;
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
    // With an append, the rows are stored once the item's first chunks (up to a
    // ring's worth) are issued, and always before its last chunk.
    const bool append_here = new_tok >= 0 && w0 == 0;
    const int c_split = append_here ? min(c_end, min(stages, nchunks - 1)) : c_end;
    auto issue_range = [&](int c0, int c1) {
      if (lane == 0 && ok) {
        for (int c = c0; c < c1; ++c) {
          if (*abort_flag || !issue(c, w0)) {
            ok = false;
            break;
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
    };
    issue_range(c_begin, c_split);
    if (append_here && ok) {
      const int id = row[new_tok / BS];  // re-read: a bad id was replaced by 0 for reading only
      if (id >= 0 && id < p.num_blocks)
        fresh.store(const_cast<__half*>(p.k_cache), const_cast<__half*>(p.v_cache),
                    p.num_kv_heads, BS, kvh, id, new_tok % BS, lane);
    }
    issue_range(c_split, c_end);
    __syncwarp();  // s_ids is rewritten for the next window
  }
  return ok;
}

// After an abort only the last SPW fills of each sub-ring can still be in
// flight: let them land before this CTA's shared memory can be handed to
// another CTA.
__device__ __forceinline__ void drain_ring(uint64_t* bars, int stages, const RingFills& issued) {
  const int spw = stages / NW;
  for (int w = 0; w < NW; ++w)
    for (int k = max(0, issued.n[w] - spw); k < issued.n[w]; ++k)
      mbar_wait(smem_u32(&bars[ring_stage(k, w, spw)]), (k / spw) & 1);
}

// ---- consumer side ---------------------------------------------------------------

template <int D>
struct Acc {
  float m0, m1;  // running max of heads 2t, 2t+1 (log2 units)
  float l0, l1;  // this lane's part of the running sums
  float o[D / 16][4];
  __device__ __forceinline__ void reset() {
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
  }
};

// One 16-token stage: QK^T, masked online softmax, PV.  valid = rows of the
// stage inside the context (1..16).
template <int D>
__device__ __forceinline__ void consume_stage(Acc<D>& a, uint32_t kt, int valid,
                                              const uint32_t (&qb)[D / 16][2], float scale_log2,
                                              int lane) {
  using Geo = StageGeom<D>;
  const uint32_t vt = kt + Geo::TILE_BYTES;
  const int g = lane >> 2;
  const int mat = lane >> 3;  // ldmatrix: which 8x8 matrix this lane addresses
  const int r8 = lane & 7;    // ... and which of its rows

  // ---- S^T = K . Q^T ----
  float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int ks = 0; ks < Geo::MT; ++ks) {
    const int tok = r8 + ((mat & 1) << 3);
    const int colh = ks * 16 + ((mat >> 1) << 3);
    uint32_t a0, a1, a2, a3;
    ldmatrix_x4(swz_addr(kt, tok, colh), a0, a1, a2, a3);
    mma_16816(sc, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
  }
  const float s0 = g < valid ? sc[0] * scale_log2 : -INFINITY;
  const float s1 = g < valid ? sc[1] * scale_log2 : -INFINITY;
  const float s2 = g + 8 < valid ? sc[2] * scale_log2 : -INFINITY;
  const float s3 = g + 8 < valid ? sc[3] * scale_log2 : -INFINITY;
  float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
  }
  const float mn0 = fmaxf(a.m0, mx0), mn1 = fmaxf(a.m1, mx1);  // finite: row 0 is valid
  const float al0 = rescale_factor(a.m0, mn0), al1 = rescale_factor(a.m1, mn1);
  a.m0 = mn0;
  a.m1 = mn1;
  const uint32_t p01 = pack_half2(exp2f(s0 - mn0), exp2f(s1 - mn1));  // token g
  const uint32_t p23 = pack_half2(exp2f(s2 - mn0), exp2f(s3 - mn1));  // token g + 8
  const float2 f01 = unpack_half2(p01), f23 = unpack_half2(p23);
  a.l0 = fmaf(a.l0, al0, f01.x + f23.x);
  a.l1 = fmaf(a.l1, al1, f01.y + f23.y);
#pragma unroll
  for (int mt = 0; mt < Geo::MT; ++mt) {
    a.o[mt][0] *= al0;
    a.o[mt][1] *= al1;
    a.o[mt][2] *= al0;
    a.o[mt][3] *= al1;
  }
  // P^T fragments: {P[token 2t][head g], P[token 2t+1][head g]} (+8 for pb1)
  const uint32_t pb0 = movmatrix_trans(p01);
  const uint32_t pb1 = movmatrix_trans(p23);
  const bool partial = valid < CHUNK;
  if (partial) {
    // Zero the V rows past the context (whole 128-byte rows, so the swizzle
    // does not matter).
    const int rows = CHUNK - valid;
    for (int idx = lane; idx < rows * Geo::NSL * 8; idx += 32) {
      const int r = valid + idx / (Geo::NSL * 8);
      const int rem = idx % (Geo::NSL * 8);
      const uint32_t addr = vt + (rem >> 3) * Geo::SLICE_BYTES + r * 128 + ((rem & 7) << 4);
      asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
    }
    __syncwarp();
  }
  // ---- O^T += V^T . P^T ----
#pragma unroll
  for (int mt = 0; mt < Geo::MT; ++mt) {
    const int tok = r8 + ((mat >> 1) << 3);
    const int colh = mt * 16 + ((mat & 1) << 3);
    uint32_t a0, a1, a2, a3;
    ldmatrix_x4_trans(swz_addr(vt, tok, colh), a0, a1, a2, a3);
    mma_16816(a.o[mt], a0, a1, a2, a3, pb0, pb1);
  }
  if (partial) fence_proxy_async_smem();  // generic writes before the next TMA fill
}

// B operand of S^T = K . Q^T from a [rows = heads][D] fp16 query tile in
// global or shared memory (generic pointer): Q[head g][16 dims of step ks],
// zero for g >= G.
template <int D>
__device__ __forceinline__ void load_q_fragments(uint32_t (&qb)[D / 16][2], const __half* q_tile,
                                                 int G, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const __half* qrow = q_tile + (size_t)g * D;
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    qb[ks][0] = g < G ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * t) : 0u;
    qb[ks][1] = g < G ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * t + 8) : 0u;
  }
}

// Same fragments when every column comes from its own row: `qrow` is this
// lane's column (lane >> 2), NULL for a zero column.
template <int D>
__device__ __forceinline__ void load_q_column(uint32_t (&qb)[D / 16][2], const __half* qrow,
                                              int lane) {
  const int t = lane & 3;
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    qb[ks][0] = qrow ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * t) : 0u;
    qb[ks][1] = qrow ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * t + 8) : 0u;
  }
}

// A warp's state into its merge buffer (after the per-head sums are reduced):
// buf[0..7] the maxima, buf[8..15] the sums, buf[16..] the [8][OSTRIDE] outputs.
template <int D>
__device__ __forceinline__ void write_state(Acc<D>& a, float* buf, int lane) {
  using Geo = StageGeom<D>;
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    a.l0 += __shfl_xor_sync(0xffffffffu, a.l0, off);
    a.l1 += __shfl_xor_sync(0xffffffffu, a.l1, off);
  }
  if (g == 0) {
    buf[2 * t] = a.m0;
    buf[2 * t + 1] = a.m1;
    buf[8 + 2 * t] = a.l0;
    buf[8 + 2 * t + 1] = a.l1;
  }
  float* so = buf + 16;
#pragma unroll
  for (int mt = 0; mt < Geo::MT; ++mt) {
    so[(2 * t) * Geo::OSTRIDE + mt * 16 + g] = a.o[mt][0];
    so[(2 * t + 1) * Geo::OSTRIDE + mt * 16 + g] = a.o[mt][1];
    so[(2 * t) * Geo::OSTRIDE + mt * 16 + g + 8] = a.o[mt][2];
    so[(2 * t + 1) * Geo::OSTRIDE + mt * 16 + g + 8] = a.o[mt][3];
  }
}

// Merges the consumer warps' states of an item's columns and stores the result:
// the fp16 output when the item covers the whole context, else the partition's
// (max, sum, unnormalised output) for the merge.
template <int D, typename ColumnRow>
__device__ __forceinline__ void store_columns(float* const (&bufs)[NW], const DecodeParams& p,
                                              int ncols, ColumnRow row_of, int part, bool whole,
                                              int prefix_slots = 0) {
  // bufs[w]: consumer warp w's state (write_state), NULL when it had no chunk of the item.
  // row_of(c): the (sequence * num_heads + head) row of column c, or -1 to skip it.
  // prefix_slots > 0 (with whole): fold in that many finished shared-prefix partials first.
  // Each thread takes 4 consecutive dims of one column.
  constexpr int PER_COL = D / 4;
  using Geo = StageGeom<D>;
  if (!whole && p.no_merge && threadIdx.x == 0) flag_error(p.err, ERR_PREFIX);  // bound too small
  for (int idx = threadIdx.x; idx < ncols * PER_COL; idx += NW * 32) {
    const int col = idx / PER_COL;
    const int d0 = (idx % PER_COL) * 4;
    const long long bh = row_of(col);
    if (bh < 0) continue;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w)
      if (bufs[w]) M = fmaxf(M, bufs[w][col]);
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    float den = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      if (!bufs[w]) continue;
      const float a = rescale_factor(bufs[w][col], M);
      const float4 o =
          *reinterpret_cast<const float4*>(bufs[w] + 16 + col * Geo::OSTRIDE + d0);
      num.x = fmaf(a, o.x, num.x);
      num.y = fmaf(a, o.y, num.y);
      num.z = fmaf(a, o.z, num.z);
      num.w = fmaf(a, o.w, num.w);
      den = fmaf(a, bufs[w][8 + col], den);
    }
    if (prefix_slots > 0) {
      const size_t base = (size_t)bh * p.num_parts;
      float M2 = M;
      for (int i = 0; i < prefix_slots; ++i) M2 = fmaxf(M2, p.ws_ml[(base + i) * 2]);
      const float a = rescale_factor(M, M2);
      num.x *= a;
      num.y *= a;
      num.z *= a;
      num.w *= a;
      den *= a;
      for (int i = 0; i < prefix_slots; ++i) {
        const float w = rescale_factor(p.ws_ml[(base + i) * 2], M2);
        const float4 o = *reinterpret_cast<const float4*>(p.ws_o + (base + i) * D + d0);
        num.x = fmaf(w, o.x, num.x);
        num.y = fmaf(w, o.y, num.y);
        num.z = fmaf(w, o.z, num.z);
        num.w = fmaf(w, o.w, num.w);
        den = fmaf(w, p.ws_ml[(base + i) * 2 + 1], den);
      }
    }
    if (whole) {
      const float inv = 1.f / den;
      *reinterpret_cast<uint2*>(p.out + (size_t)bh * D + d0) =
          make_uint2(pack_half2(num.x * inv, num.y * inv), pack_half2(num.z * inv, num.w * inv));
    } else {
      const size_t slot = (size_t)bh * p.num_parts + part;
      *reinterpret_cast<float4*>(p.ws_o + slot * D + d0) = num;
      if (d0 == 0) {
        p.ws_ml[slot * 2] = M;
        p.ws_ml[slot * 2 + 1] = den;
      }
    }
  }
}

// Merges the consumer warps' states of one item (columns = the G query heads
// of kv head kvh of sequence b) into out, or into partial slot `part`.
template <int D>
__device__ __forceinline__ void store_item(float* const (&bufs)[NW], const DecodeParams& p, int b,
                                           int kvh, int part, int G, bool whole,
                                           int prefix_slots = 0) {
  const long long row0 = (long long)b * p.num_heads + (long long)kvh * G;
  store_columns<D>(bufs, p, G, [&](int c) { return row0 + c; }, part, whole, prefix_slots);
}

// The drained ring as merge buffers, one per consumer warp (the one-CTA-per-item kernels).
template <int D>
__device__ __forceinline__ void ring_state_buffers(float* (&bufs)[NW], unsigned char* smem) {
#pragma unroll
  for (int w = 0; w < NW; ++w)
    bufs[w] = reinterpret_cast<float*>(smem) + w * StageGeom<D>::STATE_FLOATS;
}

// ---- one CTA per (sequence, kv head, partition) ---------------------------------

template <int D, int BS, bool SPLIT>
__global__ void __launch_bounds__((NW + 1) * 32)
    mma_decode_kernel(const __grid_constant__ CUtensorMap k_map,
                      const __grid_constant__ CUtensorMap v_map, const DecodeParams p) {
  using Geo = StageGeom<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int stages = p.stages;
  const uint32_t ring = smem_u32(smem);  // [stages][K tile | V tile], 1024-aligned
  int* s_ids = reinterpret_cast<int*>(smem + (size_t)stages * 2 * Geo::TILE_BYTES);  // [32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_ids + 32);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * stages);
  // merge buffers, placed over the ring once every stage has been consumed
  float* bufs[NW];
  ring_state_buffers<D>(bufs, smem);

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
    if (!SPLIT || p.seq_prefix_tokens) {
      for (int i = threadIdx.x; i < G * D; i += blockDim.x)
        p.out[((size_t)b * p.num_heads + kvh * G) * D + i] = __float2half_rn(0.f);
    }
    return;
  }
  // with a shared prefix this kernel covers the suffix [P, L) (see the CUDA-core kernel)
  bool bad_prefix = false;
  const int P = prefix_tokens_of(p.seq_prefix_tokens, b, L, BS, &bad_prefix);
  if (bad_prefix && reporter) flag_error(p.err, ERR_PREFIX);
  const int tok0 = P + part * p.part_tokens;
  if (SPLIT && part == gridDim.z - 1 && tok0 + p.part_tokens < L && threadIdx.x == 0)
    flag_error(p.err, ERR_PREFIX);  // the grid was sized below this suffix
  const int ntok = min(L, tok0 + p.part_tokens) - tok0;
  if (ntok <= 0) return;
  const int nchunks = (ntok + CHUNK - 1) / CHUNK;
  const int nblk = (ntok + BS - 1) / BS;
  const int np = (P + p.prefix_part_tokens - 1) / p.prefix_part_tokens;  // prefix slots
  const int slot_part = np + part;
  // covering a shared prefix's whole suffix: fold in the finished prefix partials here
  const bool merge_prefix = SPLIT && P > 0 && L - P <= p.part_tokens && p.fold_prefix;

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
    const int32_t* row = p.block_tables + (size_t)b * p.max_blocks + tok0 / BS;
    const int new_tok =
        (p.k_new && tok0 + ntok == L && p.context_lens[b] == L) ? ntok - 1 : -1;
    RingFills base, issued;
    base.reset();
    issued.reset();
    produce_item<D, BS>(row, nblk, nchunks, base, kvh, b, new_tok, p, s_ids, bars, stages, ring,
                        &k_map, &v_map, l2_evict_first_policy(), abort_flag, lane, issued);
    if (lane == 0 && *abort_flag) drain_ring(bars, stages, issued);
    return;
  }

  // ---------------- consumer warps ----------------
  uint32_t qb[Geo::MT][2];
  load_q_fragments<D>(qb, p.q + ((size_t)b * p.num_heads + kvh * G) * D, G, lane);
  Acc<D> a;
  a.reset();
  bool gave_up = false;  // this warp stopped before consuming all its stages
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
    consume_stage<D>(a, ring + (uint32_t)st * 2 * Geo::TILE_BYTES, min(CHUNK, ntok - c * CHUNK),
                     qb, p.scale_log2, lane);
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars[stages + st]));
  }

  // When every warp consumed all its stages, every copy has landed and the ring
  // can hold the merge buffers.  Otherwise copies may still be landing: give up
  // (the error word already says the output is invalid).
  if (named_barrier_or(1, NW * 32, gave_up)) return;
  // the merge kernel (if any) may be scheduled once every CTA got here
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  write_state<D>(a, bufs[warp], lane);
  named_barrier_sync(1, NW * 32);
  if (p.after_prefix) asm volatile("griddepcontrol.wait;" ::: "memory");  // prefix partials ready
  store_item<D>(bufs, p, b, kvh, slot_part, G,
                !SPLIT || (P == 0 && L <= p.part_tokens) || merge_prefix, merge_prefix ? np : 0);
}

// ---- shared-prefix pass ------------------------------------------------------------
//
// Sequences forked from one prompt share the prompt's blocks through their
// tables (lpnh.cn/news/2758356 §4.1-§4.2; n1n.ai "前缀缓存").  This pass reads
// such a shared prefix once for all sequences of a group: CTA = (kv head,
// group, prefix partition), and the columns of the tensor-core tile are the
// members' query heads of that kv head (member-major, G per member, at most 8
// columns), so every K/V stage feeds all members.  Each member's partial
// result goes to its prefix slots; the suffix pass covers the tokens after the
// prefix and the merge combines the two.
//
// A member is used only if its prefix length matches the group's and its table
// entries over this partition equal those of the group's first usable member;
// otherwise it is dropped from the tile and PAGEDKV_DEVERR_PREFIX is raised.

template <int D, int BS>
__global__ void __launch_bounds__((NW + 1) * 32)
    mma_prefix_kernel(const __grid_constant__ CUtensorMap k_map,
                      const __grid_constant__ CUtensorMap v_map, const DecodeParams p) {
  using Geo = StageGeom<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ int s_member[GROUP_MAX_MEMBERS];  // sequence of each member slot, -1 = none
  __shared__ int s_reject[GROUP_MAX_MEMBERS];
  const int stages = p.stages;
  const uint32_t ring = smem_u32(smem);
  int* s_ids = reinterpret_cast<int*>(smem + (size_t)stages * 2 * Geo::TILE_BYTES);  // [32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_ids + 32);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * stages);
  float* bufs[NW];  // merge buffers over the drained ring
  ring_state_buffers<D>(bufs, smem);

  // the suffix pass may start on the SMs this grid frees; it waits for this grid
  // before it reads the partial results
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kvh = blockIdx.x;
  const int grp = blockIdx.y;
  const int part = blockIdx.z;
  const int G = p.num_heads / p.num_kv_heads;
  const int max_members = 8 / G;  // columns are member-major, G heads each
  const int32_t* gd = p.groups + (size_t)grp * GROUP_WIDTH;
  const int pblocks = gd[0];
  if (pblocks <= 0 || pblocks > p.max_blocks) {
    if (threadIdx.x == 0 && kvh == 0 && part == 0) flag_error(p.err, ERR_PREFIX);
    return;
  }
  const int P = pblocks * BS;
  const int ppt = p.prefix_part_tokens;
  const int tok0 = part * ppt;
  if (part == gridDim.z - 1 && tok0 + ppt < P && threadIdx.x == 0 && kvh == 0)
    flag_error(p.err, ERR_PREFIX);  // the grid was sized below this prefix
  if (tok0 >= P) return;
  const int ntok = min(P, tok0 + ppt) - tok0;
  const int nchunks = (ntok + CHUNK - 1) / CHUNK;
  const int nblk = (ntok + BS - 1) / BS;
  const int blk0 = tok0 / BS;
  const bool reporter = kvh == 0 && part == 0;

  if (threadIdx.x < GROUP_MAX_MEMBERS) {
    const int i = threadIdx.x;
    const int m = gd[1 + i];
    bool ok = m >= 0 && m < p.num_seqs && i < max_members;
    if (ok) {
      const int L = min(p.context_lens[m], p.max_context_len);
      bool bad = false;
      ok = L > 0 && prefix_tokens_of(p.seq_prefix_tokens, m, L, BS, &bad) == P;
    }
    if (!ok && m != -1 && reporter) flag_error(p.err, ERR_PREFIX);
    s_member[i] = ok ? m : -1;
    s_reject[i] = 0;
  }
  __syncthreads();
  int first = -1;
  for (int i = 0; i < GROUP_MAX_MEMBERS && first < 0; ++i) first = s_member[i];
  if (first < 0) return;  // no usable member (uniform)
  const int32_t* ref_row = p.block_tables + (size_t)first * p.max_blocks + blk0;
  for (int idx = threadIdx.x; idx < GROUP_MAX_MEMBERS * nblk; idx += blockDim.x) {
    const int i = idx / nblk;
    const int m = s_member[i];
    if (m >= 0 && m != first && p.block_tables[(size_t)m * p.max_blocks + blk0 + idx % nblk] !=
                                    ref_row[idx % nblk])
      s_reject[i] = 1;
  }
  __syncthreads();
  if (threadIdx.x < GROUP_MAX_MEMBERS && s_reject[threadIdx.x]) {
    s_member[threadIdx.x] = -1;
    flag_error(p.err, ERR_PREFIX);
  }
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
    // ---------------- producer warp: the first usable member's table ----------------
    if (lane == 0) {
      prefetch_tensor_map(&k_map);
      prefetch_tensor_map(&v_map);
    }
    RingFills base, issued;
    base.reset();
    issued.reset();
    produce_item<D, BS>(ref_row, nblk, nchunks, base, kvh, first, -1, p, s_ids, bars, stages,
                        ring, &k_map, &v_map, l2_evict_first_policy(), abort_flag, lane, issued);
    if (lane == 0 && *abort_flag) drain_ring(bars, stages, issued);
    return;
  }

  // ---------------- consumer warps ----------------
  // this lane's query column (lane >> 2): head kvh*G + (col % G) of member col / G
  uint32_t qb[Geo::MT][2];
  {
    const int col = lane >> 2;
    const int m = s_member[col / G];
    const __half* qrow =
        m >= 0 ? p.q + ((size_t)m * p.num_heads + (size_t)kvh * G + col % G) * D : nullptr;
    load_q_column<D>(qb, qrow, lane);
  }
  Acc<D> a;
  a.reset();
  bool gave_up = false;
  for (int c = 0; c < nchunks; ++c) {
    const int st = c % stages;
    if (st % NW != warp) continue;
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
    consume_stage<D>(a, ring + (uint32_t)st * 2 * Geo::TILE_BYTES, min(CHUNK, ntok - c * CHUNK),
                     qb, p.scale_log2, lane);
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&bars[stages + st]));
  }
  if (named_barrier_or(1, NW * 32, gave_up)) return;
  write_state<D>(a, bufs[warp], lane);
  named_barrier_sync(1, NW * 32);
  store_columns<D>(
      bufs, p, max_members * G,
      [&](int c) -> long long {
        const int m = s_member[c / G];
        return m < 0 ? -1 : (long long)m * p.num_heads + (long long)kvh * G + c % G;
      },
      part, false);
}

// ---- persistent split-K kernel ---------------------------------------------------

struct PersistentArgs {
  unsigned int* ticket;          // next work item; zero at the start, zeroed by the last CTA
  unsigned long long* finished;  // (CTAs done << 32) + items they processed; likewise
  int write_zeros;         // no merge kernel may follow: write the zero outputs of empty contexts
};

// Run by one thread of each CTA once the CTA takes no more tickets, with the
// number of items the CTA processed.  The last CTA to get here zeroes both
// counters for the next launch on this workspace: every CTA has taken its last
// ticket by then, so nothing can add to them.  Without an abort the CTAs
// processed every item once and took one ticket each past the last, so any
// other count means the counters did not start at zero (some items were
// skipped).
__device__ __forceinline__ void release_counters(const PersistentArgs& pa, unsigned total,
                                                 unsigned items, bool check, unsigned* err) {
  __threadfence();
  const unsigned long long before = atomicAdd(pa.finished, (1ull << 32) | items);
  if ((before >> 32) == gridDim.x - 1) {
    const unsigned processed = (unsigned)(before & 0xffffffffull) + items;
    const unsigned taken = atomicExch(pa.ticket, 0u);
    atomicExch(pa.finished, 0ull);
    if (check && (processed != total || taken != total + gridDim.x))
      flag_error(err, ERR_INTERNAL);
    __threadfence();
  }
}

// Work item of ticket t: every full partition (part_tokens tokens) comes first,
// in (sequence, partition) order, then the partial last partitions, longest
// first (sequences sorted by their last partition's 16-token chunk count,
// descending, ties by sequence index), so the items left at the end of the
// launch are the shortest; kv head fastest.  pref_f[b] counts the full
// partitions of the sequences before b; by_tail lists the sequences with a
// partial partition in that order.  Returns (b, kvh, part, tokens).
__device__ __forceinline__ int4 item_of_ticket(int t, int num_kv_heads, int num_seqs,
                                               int part_tokens, const int* pref_f,
                                               const uint16_t* by_tail, const int* lens) {
  const int kvh = t % num_kv_heads;
  int u = t / num_kv_heads;
  const int total_f = pref_f[num_seqs];
  if (u >= total_f) {
    const int b = by_tail[u - total_f];
    const int L = lens[b];
    return make_int4(b, kvh, L / part_tokens, L % part_tokens);
  }
  // largest b with pref_f[b] <= u (non-decreasing, pref_f[0] = 0)
  int lo = 0, hi = num_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pref_f[mid] <= u) lo = mid;
    else hi = mid - 1;
  }
  return make_int4(lo, kvh, u - pref_f[lo], part_tokens);
}

constexpr int TAIL_KEYS = 64;  // partial partitions of 63+ chunks share the top key  // chunk-count keys of the partial-partition sort

// The shared-prefix pass's members of group g for one item (blocks blk0 ..
// blk0+nblk-1 of the prefix, Pg prefix tokens): bit i of the result for member
// slot i when that member is usable -- a sequence of the batch whose prefix
// length is Pg and whose table entries over these blocks equal those of the
// group's first usable member.  mem[i] gets every slot's sequence (all lanes).
// Run by a whole warp; one round of loads for the entries of all members.
template <int BS>
__device__ unsigned prefix_members(const DecodeParams& p, int g, int Pg, int blk0, int nblk,
                                   int max_members, int (&mem)[GROUP_MAX_MEMBERS], bool report,
                                   int lane) {
  const int32_t* gd = p.groups + (size_t)g * GROUP_WIDTH;
  int m = -1;
  bool ok = false;
  if (lane < GROUP_MAX_MEMBERS) {
    m = gd[1 + lane];
    ok = lane < max_members && m >= 0 && m < p.num_seqs;
    if (ok) {
      const int L = min(p.context_lens[m], p.max_context_len);
      bool bad = false;
      ok = L > 0 && prefix_tokens_of(p.seq_prefix_tokens, m, L, BS, &bad) == Pg;
    }
    if (!ok && m != -1 && report) flag_error(p.err, ERR_PREFIX);
  }
  unsigned mask = __ballot_sync(0xffffffffu, ok) & ((1u << GROUP_MAX_MEMBERS) - 1);
#pragma unroll
  for (int i = 0; i < GROUP_MAX_MEMBERS; ++i) mem[i] = __shfl_sync(0xffffffffu, m, i);
  if (mask == 0) return 0;
  const int first = mem[__ffs(mask) - 1];
  const int32_t* ref = p.block_tables + (size_t)first * p.max_blocks + blk0;
  unsigned differ = 0;  // member slots whose entries differ from the first member's
  for (int j = lane; j < nblk; j += 32) {
    const int32_t r = ref[j];
#pragma unroll
    for (int i = 0; i < GROUP_MAX_MEMBERS; ++i)
      if ((mask >> i) & 1)
        differ |= (p.block_tables[(size_t)mem[i] * p.max_blocks + blk0 + j] != r) ? 1u << i : 0u;
  }
  differ = __reduce_or_sync(0xffffffffu, differ);
  if (differ && lane == 0) flag_error(p.err, ERR_PREFIX);
  return mask & ~differ;
}

// Query fragments (as load_q_fragments) of a tile whose column c is used only when
// bit c of `cols` is set; other columns are zero.
template <int D>
__device__ __forceinline__ void load_q_masked(uint32_t (&qb)[D / 16][2], const __half* q_tile,
                                              unsigned cols, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const bool use = (cols >> g) & 1;
  const __half* qrow = q_tile + (size_t)g * D;
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    qb[ks][0] = use ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * t) : 0u;
    qb[ks][1] = use ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * t + 8) : 0u;
  }
}

// Columns of a prefix tile (member-major, G each) whose member slot is in `mask`.
__device__ __forceinline__ unsigned member_columns(unsigned mask, int G) {
  unsigned cols = 0;
  for (int c = 0; c < (8 / G) * G; ++c)
    if ((mask >> (c / G)) & 1) cols |= 1u << c;
  return cols;
}

// PREFIX = false: the decode pass (suffix pass of a shared-prefix call), rows =
// sequences.  PREFIX = true: the shared-prefix pass, rows = groups: an item is
// (group, kv head, partition of the group's prefix); the producer checks the
// members for the item (prefix length, table entries over the partition equal
// to the first usable member's; a member failing either is left out and raises
// PAGEDKV_DEVERR_PREFIX), the columns of the tile are the usable members' query
// heads of that kv head (member-major), and each member's partial state goes
// to its prefix slot `partition`.
template <int D, int BS, bool PREFIX>
__global__ void __launch_bounds__((NW + 1) * 32)
    mma_decode_persistent_kernel(const __grid_constant__ CUtensorMap k_map,
                                 const __grid_constant__ CUtensorMap v_map, const DecodeParams p,
                                 const PersistentArgs pa) {
  using Geo = StageGeom<D>;
  constexpr int AUX = GROUP_MAX_MEMBERS + 1;  // PREFIX: member mask, then the members
  constexpr uint32_t QTILE_BYTES = 8 * D * 2;
  // The 128-byte TMA swizzle needs 1024-byte aligned stages; the dynamic
  // shared memory is declared with that alignment (no slack is allocated), and
  // a CTA that finds it otherwise reports it and does nothing.
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_raw;
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) {
      flag_error(p.err, ERR_INTERNAL);
      release_counters(pa, 0, 0, false, p.err);
    }
    return;
  }
  if (PREFIX) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // suffix pass
  const int stages = p.stages;
  const int B = PREFIX ? p.num_groups : p.num_seqs;
  const uint32_t ring = smem_u32(smem);
  unsigned char* cur = smem + (size_t)stages * 2 * Geo::TILE_BYTES;
  __half* s_q = reinterpret_cast<__half*>(cur);  // [IQ][8][D]
  cur += IQ * QTILE_BYTES;
  float* s_merge = reinterpret_cast<float*>(cur);  // [NW][STATE_FLOATS]: the per-item merge
  cur += NW * Geo::STATE_FLOATS * sizeof(float);
  int4* s_item = reinterpret_cast<int4*>(cur);   // [IQ]
  cur += IQ * sizeof(int4);
  int* s_aux = reinterpret_cast<int*>(cur);      // PREFIX: [IQ][AUX] member mask, members
  if (PREFIX) cur += IQ * AUX * sizeof(int);
  int* s_lens = reinterpret_cast<int*>(cur);     // [B]
  int* pref_f = s_lens + B;                      // [B + 1]
  // [B]: rows with a partial partition (16-bit: rows < PERSISTENT_MAX_SEQS)
  uint16_t* by_tail = reinterpret_cast<uint16_t*>(pref_f + B + 1);
  int* tail_run = pref_f + B + 1 + (B + 1) / 2;  // [TAIL_KEYS]: counts, then insert positions
  int* s_num_tail = tail_run + TAIL_KEYS;        // [1]: sequences with a partial partition
  int* s_ids = s_num_tail + 1;                   // [32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      (reinterpret_cast<uintptr_t>(s_ids + 32) + 7) & ~uintptr_t(7));
  uint64_t* ifull = bars + 2 * stages;           // [IQ]: item descriptor + query tile landed
  uint64_t* iempty = ifull + IQ;                 // [IQ]: NW consumer warps done with the slot
  volatile int* abort_flag = reinterpret_cast<volatile int*>(iempty + IQ);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = p.num_heads / p.num_kv_heads;
  // the partitions this kernel's items cover (a prefix pass: the prefix's own)
  const int pt = PREFIX ? p.prefix_part_tokens : p.part_tokens;

  // per-sequence partition counts; the partial tails' chunk-count keys
  for (int k = threadIdx.x; k < TAIL_KEYS; k += blockDim.x) tail_run[k] = 0;
  __syncthreads();
  // s_lens[b]: the tokens this kernel covers -- L minus a shared prefix's tokens, or
  // (PREFIX) the group's prefix tokens
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    int L;
    if (PREFIX) {
      const int pb = p.groups[(size_t)b * GROUP_WIDTH];
      const bool ok = pb > 0 && pb <= p.max_blocks;
      if (!ok && blockIdx.x == 0) flag_error(p.err, ERR_PREFIX);
      L = ok ? pb * BS : 0;
    } else {
      L = p.context_lens[b];
      if (L > p.max_context_len || L <= 0) {
        if (blockIdx.x == 0) flag_error(p.err, ERR_CONTEXT_LEN);
        L = L <= 0 ? 0 : p.max_context_len;
      }
      bool bad_prefix = false;
      L -= L > 0 ? prefix_tokens_of(p.seq_prefix_tokens, b, L, BS, &bad_prefix) : 0;
      if (bad_prefix && blockIdx.x == 0) flag_error(p.err, ERR_PREFIX);
    }
    s_lens[b] = L;
    if (!PREFIX && L == 0 && pa.write_zeros && blockIdx.x == 0) {
      for (int i = 0; i < p.num_heads * D; ++i)
        p.out[(size_t)b * p.num_heads * D + i] = __float2half_rn(0.f);
    }
    pref_f[b + 1] = L / pt;
    const int tail = L % pt;
    if (tail) atomicAdd(&tail_run[min(TAIL_KEYS - 1, (tail + CHUNK - 1) / CHUNK)], 1);
  }
  if (threadIdx.x == 0) {
    pref_f[0] = 0;
    for (int s = 0; s < stages; ++s) {
      mbar_init(smem_u32(&bars[s]), 1);
      mbar_init(smem_u32(&bars[stages + s]), 1);
    }
    for (int s = 0; s < IQ; ++s) {
      mbar_init(smem_u32(&ifull[s]), 1);
      mbar_init(smem_u32(&iempty[s]), NW);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == 0) {
    // inclusive prefix of the full-partition counts
    int carry = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int b = b0 + lane;
      int v = b < B ? pref_f[b + 1] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += x;
      }
      if (b < B) pref_f[b + 1] = v + carry;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
    // first position of every key in descending key order
    carry = 0;
    for (int k0 = TAIL_KEYS - 32; k0 >= 0; k0 -= 32) {
      const int k = k0 + 31 - lane;  // lane 0 takes the largest key of the group
      const int c = tail_run[k];
      int v = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += x;
      }
      tail_run[k] = carry + v - c;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) *s_num_tail = carry;
    __syncwarp();
    // stable placement: sequences in index order within each key
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int b = b0 + lane;
      const int tail = b < B ? s_lens[b] % pt : 0;
      const int key = tail ? min(TAIL_KEYS - 1, (tail + CHUNK - 1) / CHUNK) : -1 - lane;
      const unsigned same = __match_any_sync(0xffffffffu, key);
      if (tail) {
        const int rank = __popc(same & ((1u << lane) - 1));
        by_tail[tail_run[key] + rank] = (uint16_t)b;
      }
      __syncwarp();
      if (tail && (same & ((1u << lane) - 1)) == 0) tail_run[key] += __popc(same);
      __syncwarp();
    }
  }
  __syncthreads();
  const int total = p.num_kv_heads * (pref_f[B] + *s_num_tail);
  // shared-prefix tokens of sequence b (0 without a prefix), as in the prologue
  auto prefix_of = [&](int b) -> int {
    if (!p.seq_prefix_tokens) return 0;
    const int L = min(p.context_lens[b], p.max_context_len);
    bool bad = false;
    return L > 0 ? prefix_tokens_of(p.seq_prefix_tokens, b, L, BS, &bad) : 0;
  };

  if (warp == NW) {
    // ---------------- producer warp ----------------
    if (lane == 0) {
      prefetch_tensor_map(&k_map);
      prefetch_tensor_map(&v_map);
    }
    const uint64_t policy = l2_evict_first_policy();
    RingFills base, issued;  // fills per consumer warp: before the next item / issued so far
    base.reset();
    issued.reset();
    // A ticket is taken when the previous item has been issued: taking them
    // earlier reserves work a CTA cannot start yet and unbalances the end.
    // (unsigned: whatever value the counter holds, a ticket is an item in range or the end)
    auto next_item = [&](int4* item) {
      const unsigned t = __shfl_sync(0xffffffffu, lane == 0 ? atomicAdd(pa.ticket, 1u) : 0u, 0);
      const bool ok = t < (unsigned)total;
      *item = ok ? item_of_ticket((int)t, p.num_kv_heads, B, pt, pref_f, by_tail, s_lens)
                 : make_int4(0, 0, 0, 0);
      return ok;
    };
    int4 d;
    bool have = next_item(&d);
    unsigned items = 0;  // items taken (lane 0's count is the one reported)
    for (int it = 0;; ++it) {
      const bool done = !have || __shfl_sync(0xffffffffu, *abort_flag, 0) != 0;
      if (done) d = make_int4(0, 0, 0, 0);
      const int qs = it % IQ;
      // (PREFIX) the item's usable members, checked before its slot is written
      unsigned mask = 0;
      int mem[GROUP_MAX_MEMBERS];
      if (PREFIX && !done)
        mask = prefix_members<BS>(p, d.x, s_lens[d.x], d.z * pt / BS, (d.w + BS - 1) / BS, 8 / G,
                                  mem, d.y == 0 && d.z == 0, lane);
      bool ok = true;
      if (lane == 0) {
        if (it >= IQ && !mbar_wait(smem_u32(&iempty[qs]), ((it / IQ) - 1) & 1)) {
          *abort_flag = 1;
          flag_error(p.err, ERR_TIMEOUT);
          ok = false;
        }
        if (ok) {
          s_item[qs] = d;
          const uint32_t full = smem_u32(&ifull[qs]);
          if (done) {
            mbar_arrive(full);  // the end marker (tokens = 0)
          } else if (PREFIX) {
            s_aux[qs * AUX] = (int)mask;
            for (int i = 0; i < GROUP_MAX_MEMBERS; ++i) s_aux[qs * AUX + 1 + i] = mem[i];
            // the usable members' query rows of kv head d.y: columns i*G .. i*G+G-1
            if (mask) {
              mbar_arrive_expect_tx(full, (uint32_t)(__popc(mask) * G * D * 2));
              for (int i = 0; i < GROUP_MAX_MEMBERS; ++i)
                if ((mask >> i) & 1)
                  bulk_load(smem_u32(s_q) + qs * QTILE_BYTES + (uint32_t)(i * G * D * 2),
                            p.q + ((size_t)mem[i] * p.num_heads + d.y * G) * D,
                            (uint32_t)(G * D * 2), full, policy);
            } else {
              mbar_arrive(full);
            }
          } else {
            mbar_arrive_expect_tx(full, (uint32_t)(G * D * 2));
            bulk_load(smem_u32(s_q) + qs * QTILE_BYTES,
                      p.q + ((size_t)d.x * p.num_heads + d.y * G) * D, (uint32_t)(G * D * 2), full,
                      policy);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
      if (done || !ok) break;
      // the item's table row, chunks and (fused append) new token
      const int nblk = (d.w + BS - 1) / BS;
      int nchunks = (d.w + CHUNK - 1) / CHUNK;
      const int32_t* row;
      int new_tok = -1;
      if (PREFIX) {
        row = p.block_tables + (size_t)mem[mask ? __ffs(mask) - 1 : 0] * p.max_blocks +
              d.z * pt / BS;
        if (!mask) nchunks = 0;  // no usable member: nothing to stream
      } else {
        const int P = prefix_of(d.x);
        row = p.block_tables + (size_t)d.x * p.max_blocks + (P + d.z * pt) / BS;
        const int Ls = s_lens[d.x];
        new_tok =
            (p.k_new && d.z * pt + d.w == Ls && p.context_lens[d.x] == P + Ls) ? d.w - 1 : -1;
      }
      if (nchunks > 0 &&
          !produce_item<D, BS>(row, nblk, nchunks, base, d.y, d.x, new_tok, p, s_ids, bars,
                               stages, ring, &k_map, &v_map, policy, abort_flag, lane, issued))
        break;
      base.advance(nchunks);
      ++items;
      have = next_item(&d);
    }
    if (lane == 0) {
      const bool aborted = *abort_flag != 0;
      if (aborted) drain_ring(bars, stages, issued);
      release_counters(pa, (unsigned)total, items, !aborted, p.err);
    }
    return;
  }

  // ---------------- consumer warps ----------------
  // (Keeping each warp's last stage of an item as its merge buffer, instead of a
  // buffer of its own, fits 6 CTAs per SM instead of 5 but measured slower.)
  const int spw = stages / NW;
  int mine = 0;  // fills of this warp's sub-ring consumed so far
  for (int it = 0;; ++it) {
    const int qs = it % IQ;
    bool stop = false, gave_up = false;
    int4 d = make_int4(0, 0, 0, 0);
    const bool ready = mbar_wait(smem_u32(&ifull[qs]), (it / IQ) & 1);
    if (!__all_sync(0xffffffffu, ready)) {
      if (lane == 0) {
        *abort_flag = 1;
        flag_error(p.err, ERR_TIMEOUT);
      }
      stop = true;
    } else {
      d = s_item[qs];
      stop = d.w == 0;
    }
    unsigned mask = 0;                 // PREFIX: usable member slots of the item
    int mem[GROUP_MAX_MEMBERS];        // PREFIX: the member slots' sequences
    if (PREFIX && !stop) {
      mask = (unsigned)s_aux[qs * AUX];
#pragma unroll
      for (int i = 0; i < GROUP_MAX_MEMBERS; ++i) mem[i] = s_aux[qs * AUX + 1 + i];
    }
    Acc<D> a;
    a.reset();
    if (!stop) {
      uint32_t qb[Geo::MT][2];
      if (PREFIX) load_q_masked<D>(qb, s_q + qs * (8 * D), member_columns(mask, G), lane);
      else load_q_fragments<D>(qb, s_q + qs * (8 * D), G, lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&iempty[qs]));  // descriptor and query tile consumed
      const int nchunks = (PREFIX && !mask) ? 0 : (d.w + CHUNK - 1) / CHUNK;
      // chunks warp, warp + NW, ... of the item: this warp's next fills, in order
      for (int j = warp; j < nchunks; j += NW, ++mine) {
        const int st = ring_stage(mine, warp, spw);
        if (__shfl_sync(0xffffffffu, *abort_flag, 0)) {
          gave_up = true;
          break;
        }
        const bool ok = mbar_wait(smem_u32(&bars[st]), (mine / spw) & 1);
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) {
            *abort_flag = 1;
            flag_error(p.err, ERR_TIMEOUT);
          }
          gave_up = true;
          break;
        }
        consume_stage<D>(a, ring + (uint32_t)st * 2 * Geo::TILE_BYTES,
                         min(CHUNK, d.w - j * CHUNK), qb, p.scale_log2, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars[stages + st]));
      }
    }
    // All consumer warps decide together: the end of the work, or an abort anywhere.
    if (named_barrier_or(1, NW * 32, stop || gave_up)) break;
    float* bufs[NW];
#pragma unroll
    for (int w = 0; w < NW; ++w) bufs[w] = s_merge + w * Geo::STATE_FLOATS;
    write_state<D>(a, s_merge + warp * Geo::STATE_FLOATS, lane);
    named_barrier_sync(1, NW * 32);
    if (PREFIX) {
      // each usable member's partial state goes to its prefix slot d.z
      const int kvh = d.y;
      store_columns<D>(
          bufs, p, (8 / G) * G,
          [&](int c) -> long long {
            const int i = c / G;
            return ((mask >> i) & 1) ? (long long)mem[i] * p.num_heads + (long long)kvh * G + c % G
                                     : -1;
          },
          d.z, false);
    } else {
      // a whole suffix (one item) is finished here, a shared prefix's partials folded in
      // (only that waits for the prefix pass)
      const int P = prefix_of(d.x);
      const int np = (P + p.prefix_part_tokens - 1) / p.prefix_part_tokens;
      const bool whole = s_lens[d.x] <= pt && (P == 0 || p.fold_prefix);
      if (whole && P > 0 && p.after_prefix) asm volatile("griddepcontrol.wait;" ::: "memory");
      store_item<D>(bufs, p, d.x, d.y, np + d.z, G, whole, whole ? np : 0);
    }
  }
  // the merge kernel may be scheduled once every CTA got here
  if (!PREFIX) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

constexpr int MAX_DEVICES = 64;

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

template <int D, int BS, bool SPLIT>
cudaError_t launch_mma_instance(const DecodeParams& p, const CUtensorMap& km,
                                const CUtensorMap& vm, cudaStream_t stream) {
  static std::atomic<int> granted[MAX_DEVICES];
  auto kernel = mma_decode_kernel<D, BS, SPLIT>;
  const size_t smem = mma_smem_bytes(D, BS, p.stages);
  cudaError_t e = allow_smem(kernel, smem, granted);
  if (e != cudaSuccess) return e;
  const dim3 grid(p.num_kv_heads, p.num_seqs, SPLIT ? p.grid_parts : 1);
  return launch_kernel(p.after_prefix != 0, kernel, grid, dim3((NW + 1) * 32), smem, stream, km,
                       vm, p);
}

template <int D, int BS, bool PREFIX>
cudaError_t launch_persistent_instance(const DecodeParams& p, const CUtensorMap& km,
                                       const CUtensorMap& vm, unsigned int* counters, bool split,
                                       long long items, cudaStream_t stream) {
  static std::atomic<int> granted[MAX_DEVICES];
  static std::atomic<int> blocks_per_sm[MAX_DEVICES];
  static std::atomic<int> blocks_smem[MAX_DEVICES];
  auto kernel = mma_decode_persistent_kernel<D, BS, PREFIX>;
  const size_t smem =
      mma_persistent_smem_bytes(D, p.stages, PREFIX ? p.num_groups : p.num_seqs, PREFIX);
  cudaError_t e = allow_smem(kernel, smem, granted);
  if (e != cudaSuccess) return e;
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
  if (blocks_smem[dev].load(std::memory_order_relaxed) != (int)smem) {
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, (NW + 1) * 32, smem);
    if (e != cudaSuccess) return e;
    blocks_per_sm[dev].store(n < 1 ? 1 : n, std::memory_order_relaxed);
    blocks_smem[dev].store((int)smem, std::memory_order_relaxed);
  }
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  // no more CTAs than work items can exist
  long long ctas = (long long)sms * blocks_per_sm[dev].load(std::memory_order_relaxed);
  if (ctas > items) ctas = items;
  if (ctas < 1) ctas = 1;
  PersistentArgs pa;
  pa.ticket = counters + (PREFIX ? 4 : 0);
  pa.finished = reinterpret_cast<unsigned long long*>(counters + (PREFIX ? 6 : 2));
  pa.write_zeros = (!PREFIX && (!split || p.seq_prefix_tokens)) ? 1 : 0;
  return launch_kernel(!PREFIX && p.after_prefix != 0, kernel, dim3((unsigned)ctas),
                       dim3((NW + 1) * 32), smem, stream, km, vm, p, pa);
}

}  // namespace

size_t mma_stage_bytes(int head_dim, int block_size) {
  (void)block_size;  // a stage is 16 tokens whatever the block size
  return 2ull * CHUNK * head_dim * sizeof(__half);
}

size_t mma_smem_bytes(int head_dim, int block_size, int stages) {
  return 1024 /* alignment slack */ + (size_t)stages * mma_stage_bytes(head_dim, block_size) +
         32 * sizeof(int) + 2ull * stages * sizeof(uint64_t) + 16;
}

size_t mma_persistent_smem_bytes(int head_dim, int stages, int num_rows, bool prefix) {
  const size_t merge = (size_t)NW * (16 + 8 * (head_dim + 4)) * sizeof(float);
  return (size_t)stages * mma_stage_bytes(head_dim, 16) + IQ * 8ull * head_dim * 2 + merge +
         IQ * sizeof(int4) + (prefix ? IQ * (GROUP_MAX_MEMBERS + 1) * sizeof(int) : 0) +
         (2ull * num_rows + 1 + (num_rows + 1) / 2 + TAIL_KEYS + 1 + 32) * sizeof(int) + 8 +
         (2ull * stages + 2 * IQ) * sizeof(uint64_t) + 16;
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

template <int D, int BS>
cudaError_t launch_prefix_instance(const DecodeParams& p, const CUtensorMap& km,
                                   const CUtensorMap& vm, int prefix_parts, cudaStream_t stream) {
  static std::atomic<int> granted[MAX_DEVICES];
  auto kernel = mma_prefix_kernel<D, BS>;
  const size_t smem = mma_smem_bytes(D, BS, p.stages);
  cudaError_t e = allow_smem(kernel, smem, granted);
  if (e != cudaSuccess) return e;
  const dim3 grid(p.num_kv_heads, p.num_groups, prefix_parts);
  kernel<<<grid, (NW + 1) * 32, smem, stream>>>(km, vm, p);
  return cudaGetLastError();
}

#define PKV_MMA_PREFIX_CASE(D_, BS_)            \
  if (p.head_dim == D_ && p.block_size == BS_) \
    return launch_prefix_instance<D_, BS_>(p, km, vm, prefix_parts, stream);

cudaError_t launch_mma_prefix(const DecodeParams& p, const CUtensorMap& km, const CUtensorMap& vm,
                              int prefix_parts, cudaStream_t stream) {
  PKV_MMA_PREFIX_CASE(64, 8)
  PKV_MMA_PREFIX_CASE(64, 16)
  PKV_MMA_PREFIX_CASE(64, 32)
  PKV_MMA_PREFIX_CASE(64, 64)
  PKV_MMA_PREFIX_CASE(128, 8)
  PKV_MMA_PREFIX_CASE(128, 16)
  PKV_MMA_PREFIX_CASE(128, 32)
  PKV_MMA_PREFIX_CASE(128, 64)
  return cudaErrorInvalidValue;
}

#define PKV_MMA_PERSISTENT_CASE(D_, BS_)                                                      \
  if (p.head_dim == D_ && p.block_size == BS_)                                               \
    return launch_persistent_instance<D_, BS_, false>(                                       \
        p, km, vm, counters, split, (long long)p.num_kv_heads * p.num_seqs * p.num_parts, stream);

cudaError_t launch_mma_decode_persistent(const DecodeParams& p, const CUtensorMap& km,
                                         const CUtensorMap& vm, unsigned int* counters, bool split,
                                         cudaStream_t stream) {
  PKV_MMA_PERSISTENT_CASE(64, 8)
  PKV_MMA_PERSISTENT_CASE(64, 16)
  PKV_MMA_PERSISTENT_CASE(64, 32)
  PKV_MMA_PERSISTENT_CASE(64, 64)
  PKV_MMA_PERSISTENT_CASE(128, 8)
  PKV_MMA_PERSISTENT_CASE(128, 16)
  PKV_MMA_PERSISTENT_CASE(128, 32)
  PKV_MMA_PERSISTENT_CASE(128, 64)
  return cudaErrorInvalidValue;
}

#define PKV_MMA_PREFIX_PERSISTENT_CASE(D_, BS_)                                             \
  if (p.head_dim == D_ && p.block_size == BS_)                                             \
    return launch_persistent_instance<D_, BS_, true>(                                      \
        p, km, vm, counters, true, (long long)p.num_kv_heads * p.num_groups * prefix_parts, stream);

cudaError_t launch_mma_prefix_persistent(const DecodeParams& p, const CUtensorMap& km,
                                         const CUtensorMap& vm, unsigned int* counters,
                                         int prefix_parts, cudaStream_t stream) {
  PKV_MMA_PREFIX_PERSISTENT_CASE(64, 8)
  PKV_MMA_PREFIX_PERSISTENT_CASE(64, 16)
  PKV_MMA_PREFIX_PERSISTENT_CASE(64, 32)
  PKV_MMA_PREFIX_PERSISTENT_CASE(64, 64)
  PKV_MMA_PREFIX_PERSISTENT_CASE(128, 8)
  PKV_MMA_PREFIX_PERSISTENT_CASE(128, 16)
  PKV_MMA_PREFIX_PERSISTENT_CASE(128, 32)
  PKV_MMA_PREFIX_PERSISTENT_CASE(128, 64)
  return cudaErrorInvalidValue;
}

}  // namespace pkv
