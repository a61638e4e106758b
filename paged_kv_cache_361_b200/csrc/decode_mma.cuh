// Paged decode attention on the tensor cores, for grouped-query heads.
//
// P2 = "PagedAttention：操作系统级 KV 缓存虚拟内存管理".
//   §1.1  out = softmax(scale * q K^T) V.
//   §3.2.2 step 4, §4.1  every logical block is visited through the block
//         table, the query group stays in registers, and the softmax is
//         accumulated tile by tile.
//   §4.2  blocks are contiguous; they are moved as whole tiles.
//
// When G = Hq / Hkv query heads share a kv head, each K/V byte feeds 2G
// multiply-adds; on the CUDA cores that (plus the bf16 unpacking and the
// cross-lane reductions) outruns the instruction issue rate before HBM is
// saturated. Here the two contractions run as m16n8k16 bf16 MMAs with a
// warp's 16 tokens (or 16 dims) as the M rows and the G heads as the N columns
// (columns G..7 are zero), so no MMA row is padding:
//   S^T = K Q^T  : A = K tile via ldmatrix, B = Q (registers, loaded once);
//   O^T += V^T P^T: A = V tile via ldmatrix.trans, B = P (the S^T accumulator
//                   transposed in registers by movmatrix, split into a bf16
//                   high part and a bf16 remainder so that P keeps ~16
//                   mantissa bits).
// K/V tiles arrive by TMA tensor copies, one cp.async.bulk.tensor.3d per
// (block, head) tile landing as [half][block_size rows][128 B] with the
// 128-byte swizzle, so the 8-row ldmatrix reads hit 8 different bank groups.
// Tokens past the context length get -inf scores and their V rows are zeroed
// in registers, so padding (even NaN) never reaches the result.
// Persistent CTAs (as many as fit on the GPU) take work items (kv head,
// sequence, partition) from an atomic counter. Warp 4 is the TMA producer: it
// walks item after item without draining the stage ring, writing a small
// descriptor per stage (which item, how many tokens, first/last chunk) and, on
// an item's first chunk, copying the item's G query rows next to the stage.
// Warps 0-3 consume (warp w owns tokens [16w, 16w+16) of each 64-token chunk);
// at an item's last chunk they fold their states into warp 0 in two rounds
// through shared memory (named barrier, producer not involved) while the
// producer keeps prefetching the next item. A split sequence's partitions are
// merged afterwards by decode_reduce_kernel.
#pragma once

#include <cuda.h>

#include "decode_common.cuh"

namespace pa {

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Fetch a tensor map's descriptor ahead of its first copy.
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// The same for a 3-D map: coordinates (x, y, z).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y, int32_t z,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// One (block, kv head) tile of K or V, [bs rows x D], into a stage: one copy
// whatever D is. At D 128 the map is 3-D (x: 64 elements = one 128-byte
// column box, y: pool row, z: which 64-element half, stride 128 bytes), so the
// copy lands as [half][row][128 B]; at D 64 it is the 2-D [row][128 B] box.
template <int D>
__device__ __forceinline__ void tma_block(uint32_t dst, const CUtensorMap* map, int32_t y, uint64_t* bar,
                                          uint64_t policy) {
  if constexpr (D == 128)
    tma_load_3d(dst, map, 0, y, 0, bar, policy);
  else
    tma_load_2d(dst, map, 0, y, bar, policy);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// p -> (bf16(p), bf16(p - bf16(p))) for a pair.
__device__ __forceinline__ void split_pair(float x, float y, uint32_t& hi, uint32_t& lo) {
  __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  const float2 hf = __bfloat1622float2(h);
  __nv_bfloat162 l = __floats2bfloat162_rn(x - hf.x, y - hf.y);
  hi = *reinterpret_cast<uint32_t*>(&h);
  lo = *reinterpret_cast<uint32_t*>(&l);
}

// Build-time tuning knobs of the one-CTA-per-item kernel (defaults measured
// on B200): ring stages at head_dim 128 (0 = the default of 2), and the CTAs
// per SM its register budget is fitted to.
#ifndef PA_MMA_STAGES
#define PA_MMA_STAGES 0
#endif
#ifndef PA_MMA_MIN_CTAS
#define PA_MMA_MIN_CTAS 0
#endif
// A minimum-CTA bound changes ptxas's register choice even when it is 1, so
// the default (0) leaves it out.
#if PA_MMA_MIN_CTAS > 0
#define PA_MMA_LAUNCH_BOUNDS(n) __launch_bounds__(n, PA_MMA_MIN_CTAS)
#else
#define PA_MMA_LAUNCH_BOUNDS(n) __launch_bounds__(n)
#endif

template <int D>
struct MmaCfg {
  static constexpr int kConsumerWarps = 4;
  static constexpr int kThreads = 32 * (kConsumerWarps + 1);
  static constexpr int kChunk = 64;                        // tokens per stage
  static constexpr int kHalves = D / 64;                   // 128-byte column boxes per row
  static constexpr int kHalfBytes = kChunk * 128;          // one 64-element column of a stage's K (or V)
  static constexpr int kTileBytes = kHalves * kHalfBytes;  // K (or V) of one stage
  static constexpr int kStageBytes = 2 * kTileBytes;
  // one-CTA-per-item kernels (and the cascade prefix pass): two 32 KB stages at
  // head_dim 128, so three CTAs share an SM (measured on B200 against three
  // stages and two CTAs: continuous batching 0.1383 -> 0.1322 ms, the cascade
  // 0.0427 -> 0.0407 ms); the persistent kernel keeps three (its producer runs
  // across items; two stages there: long context 0.2253 -> 0.2347 ms)
  static constexpr int kStages = kStageBytes <= 16384 ? 4 : (PA_MMA_STAGES > 0 ? PA_MMA_STAGES : 2);
  static constexpr int kPStages = kStageBytes <= 16384 ? 4 : 3;
  static constexpr int kQBytes = 8 * D * 2;                // query rows of one item (G <= 8)
  static constexpr int kFoldFloats = 32 * (D / 4 + 4);     // one warp's O fragments + (m, l) of 2 heads per lane
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes;  // one CTA per item
  static constexpr int kPersistSmemBytes = 1024 + kPStages * kStageBytes + kPStages * kQBytes + 2 * kFoldFloats * 4;
};


// m16n8k16 bf16 MMA, fp32 accumulate in place (all four A registers).
__device__ __forceinline__ void mma16x8(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose of an 8x8 matrix of 16-bit pairs held as MMA fragments: the lane
// holding (row i, columns 2j, 2j+1) receives (row j', ...) of the transpose.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// One consumer warp's share of a stage: its 16 tokens (nv of them valid) of
// the K tile at kst and the V tile at vst, with the tokens as the MMA's M:
//   S^T = K q^T   (M 16 tokens, N 8 heads, K 16 dims per step: 8 MMAs at D 128,
//                  in two independent chains)
//   O^T += V^T P^T (M 16 dims, N 8 heads, K 16 tokens: 2 MMAs per 16 dims,
//                  P split into a bf16 high part and remainder)
// so no MMA row is spent on padding heads (G <= 8 fill the N columns). A lane
// holds heads 2c, 2c+1 (c = lane % 4) of tokens / dims r, r + 8 (r = lane / 4);
// the running max and sum are per head; P^T's fragments come from S^T's by an
// 8x8 transpose in registers (movmatrix). V rows of invalid tokens are zeroed
// in registers so padding never reaches O.
//   o[t][0..3]: dims 16t + r (heads 2c, 2c+1), 16t + r + 8 (heads 2c, 2c+1)
template <int D>
__device__ __forceinline__ void mma_chunk(uint32_t kst, uint32_t vst, int nv, const uint32_t (&qb)[D / 16][2],
                                          float scale_log2, int lane, int warp, float (&m_run)[2], float (&l_run)[2],
                                          float (&o)[D / 16][4], int bs) {
  using Cfg = MmaCfg<D>;
  constexpr int KS = D / 16;
  const int c = lane & 3, r = lane >> 2;
  const int mk = lane >> 3, ik = lane & 7;
  // ldmatrix rows: K matrices (tok0, d0), (tok0, d0+8), (tok0+8, d0), (tok0+8, d0+8);
  // V matrices (tok0, d0), (tok0+8, d0), (tok0, d0+8), (tok0+8, d0+8)
  const int tokK = warp * 16 + (mk >> 1) * 8 + ik;
  const int dK = (mk & 1) * 8;
  const int tokV = warp * 16 + (mk & 1) * 8 + ik;
  const int dV = (mk >> 1) * 8;
  // stage layout: block b of the chunk at b * bs * D * 2 bytes, inside it the
  // 64-element half h at h * bs * 128, row t at t * 128, its 16-byte pieces
  // swizzled by (t & 7) (the 128-byte swizzle of the TMA; block and half
  // offsets are multiples of 1024 bytes, so the phase is the token's)
  const uint32_t hstride = static_cast<uint32_t>(bs) * 128u;
  const uint32_t kbase = kst + (tokK + (tokK & ~(bs - 1)) * (Cfg::kHalves - 1)) * 128;
  const uint32_t vbase = vst + (tokV + (tokV & ~(bs - 1)) * (Cfg::kHalves - 1)) * 128;
  auto k_addr = [&](int kk) {
    const int d0 = kk * 16 + dK;
    return kbase + (d0 >> 6) * hstride + ((((d0 & 63) >> 3) ^ (tokK & 7)) << 4);
  };
  auto v_addr = [&](int dgi) {
    const int d0 = dgi * 16 + dV;
    return vbase + (d0 >> 6) * hstride + ((((d0 & 63) >> 3) ^ (tokV & 7)) << 4);
  };
  float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int kk = 0; kk < KS; ++kk) {
    uint32_t m0, m1, m2, m3;
    ldsm_x4(k_addr(kk), m0, m1, m2, m3);
    // A = K rows (tokens) x 16 dims: a0 (tok0, d0), a1 (tok0+8, d0), a2 (tok0, d0+8), a3 (tok0+8, d0+8)
    mma16x8(kk & 1 ? s1 : s0, m0, m2, m1, m3, qb[kk][0], qb[kk][1]);
  }
  float x[4];
  const bool va = r < nv, vb = r + 8 < nv;
#pragma unroll
  for (int e = 0; e < 4; ++e) x[e] = (e < 2 ? va : vb) ? (s0[e] + s1[e]) * scale_log2 : -INFINITY;
  float mloc[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    float v = fmaxf(x[j], x[2 + j]);
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
    mloc[j] = v;
  }
  // the reference maximum moves only when a score exceeds it by 8 (log2
  // units): weights stay <= 2^8 and O is rarely rescaled
  bool move[2];
  float mn[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    move[j] = mloc[j] > m_run[j] + 8.f;
    mn[j] = move[j] ? mloc[j] : m_run[j];
  }
  float pr[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) pr[e] = fast_exp2(x[e] - mn[e & 1]);
  if (__any_sync(0xffffffffu, move[0] || move[1])) {
    float alpha[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      alpha[j] = fast_exp2(m_run[j] - mn[j]);  // 1 for heads that did not move, 0 from -inf
      l_run[j] *= alpha[j];
    }
#pragma unroll
    for (int t = 0; t < D / 16; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[t][e] *= alpha[e & 1];
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    m_run[j] = mn[j];
    l_run[j] += pr[j] + pr[2 + j];
  }
  // P^T as B fragments (K 16 tokens x N 8 heads): transpose the S^T-layout pairs
  uint32_t h01, l01, h23, l23;
  split_pair(pr[0], pr[1], h01, l01);
  split_pair(pr[2], pr[3], h23, l23);
  const uint32_t bh0 = movmatrix_t(h01), bh1 = movmatrix_t(h23);
  const uint32_t bl0 = movmatrix_t(l01), bl1 = movmatrix_t(l23);
  uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
  if (nv < 16) {
    mlo = (2 * c < nv ? 0x0000ffffu : 0u) | (2 * c + 1 < nv ? 0xffff0000u : 0u);
    mhi = (2 * c + 8 < nv ? 0x0000ffffu : 0u) | (2 * c + 9 < nv ? 0xffff0000u : 0u);
  }
#pragma unroll
  for (int dgi = 0; dgi < D / 16; ++dgi) {
    uint32_t v0, v1, v2, v3;
    ldsm_x4_t(v_addr(dgi), v0, v1, v2, v3);
    // A = V^T (16 dims x 16 tokens): a0 (d0, tok0), a1 (d0+8, tok0), a2 (d0, tok0+8), a3 (d0+8, tok0+8)
    v0 &= mlo;
    v1 &= mhi;
    v2 &= mlo;
    v3 &= mhi;
    mma16x8(o[dgi], v0, v2, v1, v3, bh0, bh1);
    mma16x8(o[dgi], v0, v2, v1, v3, bl0, bl1);
  }
}

// A warp's l, summed over its lanes' tokens (lanes of one c hold the same heads).
__device__ __forceinline__ void sum_l(float (&l)[2]) {
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    l[j] += __shfl_xor_sync(0xffffffffu, l[j], 4);
    l[j] += __shfl_xor_sync(0xffffffffu, l[j], 8);
    l[j] += __shfl_xor_sync(0xffffffffu, l[j], 16);
  }
}

// Q rows (bf16, row stride D) as the B fragments of S^T = K q^T (column r =
// head r): b0 = dims (kk*16 + 2c, +1), b1 = dims +8; heads >= G are zero.
template <int D, int G>
__device__ __forceinline__ void load_q_frags(const uint32_t* qrow_words, int r, int c, uint32_t (&qa)[D / 16][2],
                                             bool from_global) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    if (r < G) {
      qa[kk][0] = from_global ? __ldg(qrow_words + kk * 8 + c) : qrow_words[kk * 8 + c];
      qa[kk][1] = from_global ? __ldg(qrow_words + kk * 8 + 4 + c) : qrow_words[kk * 8 + 4 + c];
    } else {
      qa[kk][0] = qa[kk][1] = 0u;
    }
  }
}

constexpr int kDescFirst = 1, kDescLast = 2, kDescTerm = 4;

struct StageDesc {
  int32_t s, g, p, ntok, nparts, flags;
};

template <int S>
struct PersistSmem {
  uint64_t full[S];
  uint64_t empty[S];
  uint64_t cbar;  // consumer-warp barrier (one arrival per consumer warp)
  StageDesc desc[S];
  int abort_flag;
  int merge_here;  // the item just finished completes its (sequence, kv head): merge it
};

// Barrier over the consumer warps built on an mbarrier, so that its wait is
// bounded like every other wait: it gives up (false) once the CTA aborts.
__device__ __forceinline__ bool consumer_sync(uint64_t* bar, uint32_t& phase, volatile int* abort_flag, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
  const bool ok = pipe_wait(bar, phase, abort_flag);
  phase ^= 1u;
  return ok;
}

// Fold another warp's (m, l, o) (same fragment layout) into this lane's:
// per head j of the lane (o[t][j], o[t][2 + j]).
template <int D>
__device__ __forceinline__ void fold_state(float (&m)[2], float (&l)[2], float (&o)[D / 16][4], const float* src) {
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const float m2 = src[D / 4 + j], l2 = src[D / 4 + 2 + j];
    const float M = fmaxf(m[j], m2);
    if (M == -INFINITY) continue;  // both empty
    const float f1 = exp2f(m[j] - M), f2 = exp2f(m2 - M);
    l[j] = l[j] * f1 + l2 * f2;
#pragma unroll
    for (int t = 0; t < D / 16; ++t) {
      o[t][j] = o[t][j] * f1 + src[4 * t + j] * f2;
      o[t][2 + j] = o[t][2 + j] * f1 + src[4 * t + 2 + j] * f2;
    }
    m[j] = M;
  }
}

template <int D>
__device__ __forceinline__ void store_state(float* dst, const float (&m)[2], const float (&l)[2],
                                            const float (&o)[D / 16][4]) {
#pragma unroll
  for (int t = 0; t < D / 16; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) dst[4 * t + e] = o[t][e];
  dst[D / 4] = m[0];
  dst[D / 4 + 1] = m[1];
  dst[D / 4 + 2] = l[0];
  dst[D / 4 + 3] = l[1];
}

template <int D, int G>
__global__ void __launch_bounds__(MmaCfg<D>::kThreads) decode_mma_persistent_kernel(const __grid_constant__ CUtensorMap tmk,
                                                                        const __grid_constant__ CUtensorMap tmv,
                                                                        const DecodeArgs a) {
  using Cfg = MmaCfg<D>;
  constexpr int NW = Cfg::kConsumerWarps, C = Cfg::kChunk, S = Cfg::kPStages;
  static_assert(G <= 8, "query heads of one group must fit in MMA rows 0..7");

  extern __shared__ uint8_t smem_raw[];
  __shared__ PersistSmem<S> ps;
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;  // 1024-aligned: swizzle atoms
  uint8_t* sgen = smem_raw + (sbase - sraw);
  const uint32_t qslot0 = sbase + S * Cfg::kStageBytes;
  const uint8_t* qslot_gen = sgen + S * Cfg::kStageBytes;
  float* fold = reinterpret_cast<float*>(sgen + S * Cfg::kStageBytes + S * Cfg::kQBytes);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = lane >> 2, c = lane & 3;

  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < S; ++i) {
      mbar_init(&ps.full[i], 1);
      mbar_init(&ps.empty[i], NW);
    }
    mbar_init(&ps.cbar, NW);
    ps.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == NW) {
    // ------------------------------ producer ------------------------------
    const uint32_t box_bytes = static_cast<uint32_t>(a.bs) * D * 2u;  // one (block, head) tile of K or V
    const uint64_t pol = kv_stream_policy();
    const __nv_bfloat16* qbase = static_cast<const __nv_bfloat16*>(a.q);
    int item = blockIdx.x;
    int cs = 0;
    bool aborted = false;
    while (!aborted && item < a.n_items) {
      unsigned nxt = 0;
      if (lane == 0) nxt = atomicAdd(a.counters, 1u);  // next item, used at the end of this one
      int g, s, p;
      item_coords(a, item, g, s, p);
      const int32_t L = load_len(a, s, g == 0 && p == 0 && lane == 0);
      const int32_t sst = seq_start(a, s, L);
      const int32_t span = L - sst;
      const int32_t P = a.part_tokens > 0 ? a.part_tokens : (span > 0 ? span : 1);
      const int32_t t0 = sst + p * P;
      if (L == 0 && !a.starts) {
        if (p == 0)
          for (int idx = lane; idx < G * D; idx += 32)
            a.out[(static_cast<int64_t>(s) * a.hq + g * G) * D + idx] = 0.f;
      } else if (t0 < L) {
        const int32_t t1 = min(t0 + P, L);
        const int nch = (t1 - t0 + C - 1) / C;
        // fused KV append: the new row is loaded now and stored before the
        // item's last chunk's copies, which read it
        const bool do_append = a.slot_mapping && t1 == L;
        AppendRow<__nv_bfloat16, D> ar;
        if (do_append) ar.load(a, s, g, lane);
        const int nparts = a.part_tokens > 0 ? (span + P - 1) / P : 1;
        const int64_t table_row = static_cast<int64_t>(s) * a.max_blocks;
        // block ids of chunk ch (lane < its block count), loaded one chunk
        // ahead so that the table read overlaps the wait for a free stage
        auto chunk_ids = [&](int ch) -> int32_t {
          const int32_t c0 = t0 + ch * C;
          const int32_t nb = (min(C, t1 - c0) + a.bs - 1) / a.bs;  // <= 8 (bs >= 8)
          return lane < nb ? __ldg(a.tables + table_row + c0 / a.bs + lane) : -1;
        };
        int32_t blk_next = chunk_ids(0);
        for (int ch = 0; ch < nch; ++ch, ++cs) {
          const int st = cs % S;
          const int32_t blk = blk_next;
          if (ch + 1 < nch) blk_next = chunk_ids(ch + 1);
          if (cs >= S && !pipe_wait(&ps.empty[st], ((cs / S) - 1) & 1, &ps.abort_flag)) {
            aborted = true;
            break;
          }
          if (do_append) ar.before_chunk(a, ch, nch, lane);
          const int32_t c0 = t0 + ch * C;
          const int32_t n = min(C, t1 - c0);
          const int32_t nb = (n + a.bs - 1) / a.bs;  // <= 8 (bs >= 8)
          bool ok = false;
          if (lane < nb) {
            ok = blk >= 0 && blk < a.num_blocks;
            if (!ok) record_error(PA_ERR_DEVICE_BOUNDS, blk);
          }
          const unsigned okmask = __ballot_sync(0xffffffffu, ok);
          if (lane == 0) {
            StageDesc& d = ps.desc[st];
            d.s = s;
            d.g = g;
            d.p = p;
            d.ntok = n;
            d.nparts = nparts;
            d.flags = (ch == 0 ? kDescFirst : 0) | (ch == nch - 1 ? kDescLast : 0);
            const uint32_t qbytes = ch == 0 ? static_cast<uint32_t>(G * D * 2) : 0u;
            mbar_arrive_expect_tx(&ps.full[st], 2u * __popc(okmask) * box_bytes + qbytes);
            if (ch == 0)
              bulk_g2s(sgen + S * Cfg::kStageBytes + st * Cfg::kQBytes,
                       qbase + (static_cast<int64_t>(s) * a.hq + g * G) * D, qbytes, &ps.full[st], pol);
          }
          __syncwarp();
          if (ok) {
            const int32_t y = (blk * a.hkv + g) * a.bs;
            const uint32_t kdst = sbase + st * Cfg::kStageBytes + lane * box_bytes;
            tma_block<D>(kdst, &tmk, y, &ps.full[st], pol);
            tma_block<D>(kdst + Cfg::kTileBytes, &tmv, y, &ps.full[st], pol);
          }
          if (do_append) ar.after_chunk(a, ch, nch, lane);
        }
      }
      item = static_cast<int>(gridDim.x + __shfl_sync(0xffffffffu, nxt, 0));
    }
    if (!aborted) {
      const int st = cs % S;
      if (cs >= S && !pipe_wait(&ps.empty[st], ((cs / S) - 1) & 1, &ps.abort_flag)) {
        aborted = true;
      } else if (lane == 0) {
        ps.desc[st].flags = kDescTerm;
        mbar_arrive(&ps.full[st]);
      }
      ++cs;
    }
    if (aborted && lane == 0)
      for (int j = (cs > S ? cs - S : 0); j < cs; ++j) mbar_wait(&ps.full[j % S], (j / S) & 1);
    return;
  }

  // -------------------------------- consumers --------------------------------
  uint32_t qa[D / 16][2];
  float o[D / 16][4];
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  uint32_t cphase = 0;
#define PA_CSYNC()                                                    \
  do {                                                                \
    if (!consumer_sync(&ps.cbar, cphase, &ps.abort_flag, lane)) return; \
  } while (0)
#pragma unroll
  for (int t = 0; t < D / 16; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;

  for (int cs = 0;; ++cs) {
    const int st = cs % S;
    if (!pipe_wait(&ps.full[st], (cs / S) & 1, &ps.abort_flag)) return;
    const volatile StageDesc& vd = ps.desc[st];
    const int flags = vd.flags;
    if (flags & kDescTerm) return;
    const int ds = vd.s, dg = vd.g, dp = vd.p, dn = vd.ntok, dnp = vd.nparts;

    if (flags & kDescFirst) {
      load_q_frags<D, G>(reinterpret_cast<const uint32_t*>(qslot_gen + st * Cfg::kQBytes) + r * (D / 2), r, c, qa,
                         false);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        m_run[j] = -INFINITY;
        l_run[j] = 0.f;
      }
#pragma unroll
      for (int t = 0; t < D / 16; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
    }

    const int nv = min(16, dn - warp * 16);  // warp-uniform
    if (nv > 0) {
      const uint32_t kst = sbase + st * Cfg::kStageBytes;
      mma_chunk<D>(kst, kst + Cfg::kTileBytes, nv, qa, a.scale_log2, lane, warp, m_run, l_run, o, a.bs);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&ps.empty[st]);

    if (!(flags & kDescLast)) continue;

    // ---- item finished: fold warps 3,2 -> 1,0 -> 0 (two rounds), then store ----
    float lrow[2] = {l_run[0], l_run[1]};
    sum_l(lrow);
    float* slot0 = fold + lane * (D / 4 + 4);
    float* slot1 = fold + Cfg::kFoldFloats + lane * (D / 4 + 4);
    if (warp >= 2) store_state<D>(warp == 2 ? slot0 : slot1, m_run, lrow, o);
    PA_CSYNC();
    if (warp < 2) fold_state<D>(m_run, lrow, o, warp == 0 ? slot0 : slot1);
    PA_CSYNC();
    if (warp == 1) store_state<D>(slot0, m_run, lrow, o);
    PA_CSYNC();
    if (warp == 0) fold_state<D>(m_run, lrow, o, slot0);

    const int64_t row0 = static_cast<int64_t>(ds) * a.hq + dg * G;
    if (dnp == 1 && !a.force_partials) {
      if (warp == 0) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          if (2 * c + j >= G) continue;
          const float inv = 1.f / lrow[j];
          float* dst = a.out + (row0 + 2 * c + j) * D + r;
#pragma unroll
          for (int t = 0; t < D / 16; ++t) {
            dst[16 * t] = o[t][j] * inv;
            dst[16 * t + 8] = o[t][2 + j] * inv;
          }
        }
      }
      PA_CSYNC();  // the fold slots are free again
      continue;
    }
    // split sequence: publish this partition's (m, l, o); the last partition's
    // consumers (fused merge) or decode_reduce_kernel merge them
    if (warp == 0) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        if (2 * c + j >= G) continue;
        const int64_t prow = (row0 + 2 * c + j) * a.parts_stride + dp;
        float* dst = a.ws_o + prow * D + r;
#pragma unroll
        for (int t = 0; t < D / 16; ++t) {
          dst[16 * t] = o[t][j];
          dst[16 * t + 8] = o[t][2 + j];
        }
        if (r == 0) *reinterpret_cast<float2*>(a.ws_ml + prow * 2) = make_float2(m_run[j], lrow[j]);
      }
    }
    if (a.fuse_merge) {
      __threadfence();
      PA_CSYNC();
      if (warp == 0 && lane == 0) ps.merge_here = count_arrival(a, ds, dg, dnp);
      PA_CSYNC();
      if (ps.merge_here) merge_partials_to_out<G, D>(a, ds, dg * G, dnp, tid, 32 * NW);
    }
    PA_CSYNC();  // the fold slots are free again
  }
#undef PA_CSYNC
}

// One CTA per work item (kv head, sequence, partition); grid (Hkv, B, parts),
// partition-major dispatch. The producer warp streams the item's chunks; at the
// end every warp's (m, l, o) goes through shared memory (the stage ring is free
// by then) and the CTA stores the row or the partition's partials.
template <int D, int G>
__global__ void PA_MMA_LAUNCH_BOUNDS(MmaCfg<D>::kThreads) decode_mma_kernel(const __grid_constant__ CUtensorMap tmk,
                                                                        const __grid_constant__ CUtensorMap tmv,
                                                                        const DecodeArgs a) {
  using Cfg = MmaCfg<D>;
  constexpr int NW = Cfg::kConsumerWarps, C = Cfg::kChunk, S = Cfg::kStages;
  static_assert(NW * G * (D + 2) * 4 <= S * Cfg::kStageBytes, "merge buffer must fit in the stage ring");

  extern __shared__ uint8_t smem_raw[];
  __shared__ PipeSmem<S> ps;
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));

  const int g = blockIdx.x, p = blockIdx.z;
  const int s = grid_seq(a, blockIdx.y, g == 0 && p == 0 && threadIdx.x == 0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = lane >> 2, c = lane & 3;
  Part pt;
  if (!cta_part<G, D>(a, g, s, p, tid, Cfg::kThreads, pt)) return;
  const int nchunks = (pt.ntok + C - 1) / C;
  const int hq0 = g * G;

  // the producer's global reads (its first block-table window; with the fused
  // KV append the new row, stored before the last chunk's copies, which read
  // it) go out before the CTA-wide barrier
  const bool do_append = a.slot_mapping && pt.last;
  AppendRow<__nv_bfloat16, D> ar;
  TableAhead ta;
  if (warp == NW) {
    if (do_append) ar.load(a, s, g, lane);
    ta.init(a.tables + static_cast<int64_t>(s) * a.max_blocks, pt.t0 / a.bs,
            min(a.max_blocks, (pt.t1 + a.bs - 1) / a.bs), lane);
  }
  if (tid == 0) {
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
    pipe_init<S>(ps, NW);
  }
  __syncthreads();

  float o[D / 16][4];
#pragma unroll
  for (int t = 0; t < D / 16; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

  if (warp == NW) {
    const uint32_t box_bytes = static_cast<uint32_t>(a.bs) * D * 2u;  // one (block, head) tile of K or V
    const uint64_t pol = kv_stream_policy();
    pipe_produce<S>(ps, nchunks, [&](int i, int st) {
      if (do_append) ar.before_chunk(a, i, nchunks, lane);
      const int32_t c0 = pt.t0 + i * C;
      const int32_t nb = (min(C, pt.t1 - c0) + a.bs - 1) / a.bs;  // <= 8 (bs >= 8)
      const int32_t blk = ta.get(c0 / a.bs, nb, lane);
      bool ok = false;
      if (lane < nb) {
        ok = blk >= 0 && blk < a.num_blocks;
        if (!ok) record_error(PA_ERR_DEVICE_BOUNDS, blk);
      }
      const unsigned okmask = __ballot_sync(0xffffffffu, ok);
      if (lane == 0) mbar_arrive_expect_tx(&ps.full[st], 2u * __popc(okmask) * box_bytes);
      __syncwarp();
      if (ok) {
        const int32_t y = (blk * a.hkv + g) * a.bs;
        const uint32_t kdst = sbase + st * Cfg::kStageBytes + lane * box_bytes;
        tma_block<D>(kdst, &tmk, y, &ps.full[st], pol);
        tma_block<D>(kdst + Cfg::kTileBytes, &tmv, y, &ps.full[st], pol);
      }
      if (do_append) ar.after_chunk(a, i, nchunks, lane);
    });
  } else {
    uint32_t qa[D / 16][2];
    load_q_frags<D, G>(reinterpret_cast<const uint32_t*>(static_cast<const __nv_bfloat16*>(a.q) +
                                                         (static_cast<int64_t>(s) * a.hq + hq0 + (r < G ? r : 0)) * D),
                       r, c, qa, true);
    for (int i = 0; i < nchunks; ++i) {
      const int st = i % S;
      if (!pipe_wait(&ps.full[st], (i / S) & 1, &ps.abort_flag)) break;
      const int nv = min(16, min(C, pt.ntok - i * C) - warp * 16);  // warp-uniform
      if (nv > 0) {
        const uint32_t kst = sbase + st * Cfg::kStageBytes;
        mma_chunk<D>(kst, kst + Cfg::kTileBytes, nv, qa, a.scale_log2, lane, warp, m_run, l_run, o, a.bs);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ps.empty[st]);
    }
    sum_l(l_run);
  }

  __syncthreads();  // every copy consumed; the stage ring is free
  if (ps.abort_flag) return;

  float* wm = reinterpret_cast<float*>(sgen);
  float* wl = wm + NW * G;
  float* wacc = wl + NW * G;
  if (warp < NW) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int h = 2 * c + j;
      if (h >= G) continue;
      if (r == 0) {
        wm[warp * G + h] = m_run[j];
        wl[warp * G + h] = l_run[j];
      }
#pragma unroll
      for (int t = 0; t < D / 16; ++t) {
        wacc[(warp * G + h) * D + 16 * t + r] = o[t][j];
        wacc[(warp * G + h) * D + 16 * t + r + 8] = o[t][2 + j];
      }
    }
  }
  __syncthreads();
  merge_warps_and_store<G, D, NW>(a, wm, wl, wacc, s, p, hq0, pt.nparts, pt.npre, tid, Cfg::kThreads);
}

}  // namespace pa
