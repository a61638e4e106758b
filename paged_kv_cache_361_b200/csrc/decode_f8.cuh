// Paged decode attention over an 8-bit (e4m3 or int8) KV cache, on the tensor
// cores. The two formats differ only in the widening of four codes to two
// f16x2 words (widen4<CF>): conversion instructions for e4m3, byte permutes
// and one f16x2 subtraction for int8; the text below says e4m3 for both.
//
// P2 = "PagedAttention：操作系统级 KV 缓存虚拟内存管理".
//   §1.1  out = softmax(scale * q K^T) V.
//   §3.2.2 step 4, §4.1  every logical block is visited through the block
//         table; the softmax is accumulated chunk by chunk.
// P3 = "PagedAttention 和 vLLM", the section on its future: paged KV storage
//   combined with quantisation. A code c stands for value(c) * scale, one
//   scale per tensor.
//
// Half the bytes of a bf16 cache per token, so the conversion work per byte
// doubles; widening every element to fp32 on the CUDA cores runs out of
// conversion throughput long before HBM does. Here each element is widened
// once, two at a time (cvt e4m3x2 -> f16x2, exact), straight into the operand
// registers of m16n8k16 f16 MMAs with fp32 accumulation:
//   S = Q K^T : A = q (bf16 -> f16, exact for |q| < 65504) in registers,
//               B = K from shared memory with one 32-bit load per thread per
//               16 dims. The 16 dims a k-step contracts are taken in the
//               order that makes a thread's two B registers four adjacent
//               bytes (dims 4c..4c+3 of the step); Q uses the same order.
//   O += P V  : A = P as f16 (11 mantissa bits: one MMA, no split), B = V.
//               Thread (g, c) feeds output columns 16g + j (D 128; 8g + j at
//               D 64) of n-tile j, so it reads one 16-byte (8-byte) piece of
//               each of its four tokens' V rows and pairs tokens with byte
//               permutes before widening.
// K/V tiles arrive as TMA tensor copies of [block_size rows x D bytes] with
// the 128-byte (D 128) or 64-byte (D 64) swizzle, so the row-strided loads
// above are free of bank conflicts (D 128). The K scale is folded into the
// score scale, the V scale multiplies O before the merge. Tokens past the
// context length get -inf scores and zeroed V operands (their bytes may be
// NaN codes), as in the other decode kernels.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>

#include "decode_common.cuh"
#include "decode_mma.cuh"

namespace pa {

// Build-time tuning knobs, defaults measured on B200 (e4m3 metric workload):
// 3 stages and the register budget fitted to 4 CTAs per SM (q fragments read
// from shared memory at every k-step, V one 32-bit word at a time; with q in
// registers, 4 stages and 3 CTAs per SM the kernel was 5 % slower).
#ifndef PA_F8_MIN_CTAS
#define PA_F8_MIN_CTAS 4
#endif
#ifndef PA_F8_STAGES
#define PA_F8_STAGES 3
#endif
// A minimum-CTA bound changes ptxas's register choice even when it is 1, so
// 0 leaves it out.
#if PA_F8_MIN_CTAS > 0
#define PA_F8_LAUNCH_BOUNDS(n) __launch_bounds__(n, PA_F8_MIN_CTAS)
#else
#define PA_F8_LAUNCH_BOUNDS(n) __launch_bounds__(n)
#endif

template <int D>
struct F8Cfg {
  static constexpr int kConsumerWarps = 4;
  static constexpr int kThreads = 32 * (kConsumerWarps + 1);
  static constexpr int kChunk = 64;                 // tokens per stage
  static constexpr int kTileBytes = kChunk * D;     // K (or V) of one stage
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStages = PA_F8_STAGES;
  static constexpr int kQSmemBytes = 32 * (D / 16) * 8;  // q fragments of every lane
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kQSmemBytes;
};

// Byte offset of (row, byte column) in a swizzled tile of D-byte rows, as the
// TMA writes it: 16-byte chunk index XOR the row's position in the swizzle
// atom (128-byte swizzle: row & 7; 64-byte swizzle: (row >> 1) & 3).
template <int D>
__device__ __forceinline__ uint32_t f8_off(int row, int col) {
  if (D == 128) return row * 128 + ((((col >> 4) ^ (row & 7)) << 4) | (col & 15));
  return row * 64 + ((((col >> 4) ^ ((row >> 1) & 3)) << 4) | (col & 15));
}

// Four e4m3 codes (low byte first) -> two f16x2 words: bytes 0,1 -> lo,
// bytes 2,3 -> hi (low byte in the low half), exact.
__device__ __forceinline__ void e4m3x4_f16x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

// Four int8 codes (low byte first) -> two f16x2 words, paired as
// e4m3x4_f16x2 does, exact: each byte, biased by 128, becomes the low byte of
// the f16 1024 (whose unit is 1), and 1152 is subtracted.
__device__ __forceinline__ void s8x4_f16x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t u = w ^ 0x80808080u;
  const uint32_t l = __byte_perm(u, 0x64646464u, 0x5140), h = __byte_perm(u, 0x64646464u, 0x7362);
  asm("sub.f16x2 %0, %1, %2;" : "=r"(lo) : "r"(l), "r"(0x64806480u));
  asm("sub.f16x2 %0, %1, %2;" : "=r"(hi) : "r"(h), "r"(0x64806480u));
}

// Four codes of format CF -> two f16x2 words (bytes 0,1 -> lo; 2,3 -> hi).
template <int CF>
__device__ __forceinline__ void widen4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  if constexpr (CF == kCodeS8)
    s8x4_f16x2(w, lo, hi);
  else
    e4m3x4_f16x2(w, lo, hi);
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// One row of a 64-key chunk of codes, half of its dims, widened to f16. src:
// the chunk's codes as the TMA stages them ([rows x D] bytes, 128-byte swizzle
// at D 128, 64-byte at D 64); dst: the 128-byte-swizzled [rows x 64] f16 box
// columns, kHalfBytes apart, that a bf16 tile has after its TMA copy. live =
// false writes zeros (rows past the last key: their bytes may be anything).
template <int D, int CF, int kHalfBytes>
__device__ __forceinline__ void widen_row_half(const uint8_t* src, uint8_t* dst, int row, int half, bool live) {
  constexpr int DH = D / 2;  // dims per thread
  const int key = D == 128 ? (row & 7) : ((row >> 1) & 3);  // swizzle of the staged code row
  src += row * D;
  dst += row * 128;
  // every load of the row's codes first (all in flight together), then the stores
  uint4 wv[DH / 16];
#pragma unroll
  for (int u0 = 0; u0 < DH / 16; ++u0) {
    const int u = D == 128 && half ? (u0 ^ 2) : u0;
    const int d0 = half * DH + 16 * u;
    wv[u0] = live ? *reinterpret_cast<const uint4*>(src + (((d0 >> 4) ^ key) << 4)) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int u0 = 0; u0 < DH / 16; ++u0) {
    // at D 128 the two halves of a row would store to the same 16-byte columns
    // at once (lanes 2r and 2r+1 share a store phase); half 1 takes its
    // pieces in rotated order, so a phase hits 8 columns
    const int u = D == 128 && half ? (u0 ^ 2) : u0;
    const int d0 = half * DH + 16 * u;  // 16 codes -> dims d0 .. d0 + 15
    const uint4 w = wv[u0];
    uint32_t h[8];
    widen4<CF>(w.x, h[0], h[1]);
    widen4<CF>(w.y, h[2], h[3]);
    widen4<CF>(w.z, h[4], h[5]);
    widen4<CF>(w.w, h[6], h[7]);
    // two 16-byte pieces of the 128-byte row of box column d0 / 64
    uint8_t* rp = dst + (d0 >> 6) * kHalfBytes;
    const int cc = (d0 & 63) >> 3;
    *reinterpret_cast<uint4*>(rp + ((cc ^ (row & 7)) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4*>(rp + (((cc + 1) ^ (row & 7)) << 4)) = make_uint4(h[4], h[5], h[6], h[7]);
  }
}

// m16n8k16 f16 MMA, fp32 accumulate in place (all four A registers).
__device__ __forceinline__ void mma16x8_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The q fragments of a lane for k-step kk, read from shared memory (every
// consumer warp uses the same ones: 32 lanes' pairs per k-step).
struct QFragSmem {
  const uint2* p;
  int lane;
  __device__ __forceinline__ uint2 operator()(int kk) const { return p[kk * 32 + lane]; }
};

// Output dim of row r (r < 8) of m-tile t in f8_chunk's O^T, and of row r + 8
// one more: a lane's rows cover dims [16r, 16r + 16) at head_dim 128 ([8r,
// 8r + 8) at 64), which are the bytes of the one V piece it reads per token.
template <int D>
__device__ __forceinline__ int f8_dim(int t, int r) {
  return (D == 128 ? 16 : 8) * r + 2 * t;
}

// One consumer warp's 16 tokens (nv valid) of a stage, with the tokens (or
// dims) as the MMA's M and the heads as its N:
//   S^T = K q^T : A = the warp's K rows widened to f16; per k-step a thread's
//                 registers are four adjacent codes of one row, dims
//                 (16kk + 4c, +1) and (16kk + 4c + 2, +3) (one 32-bit shared
//                 load per row), q is taken in the same order; two chains
//   O^T += V^T P^T: A = V^T widened, M row r of m-tile t being dim
//                 f8_dim(t, r) (r + 8: one more), so that a thread's rows of
//                 every m-tile come from one piece of each of its four tokens'
//                 V rows, paired across tokens by byte permutes; B = P^T, the
//                 f16 weights of S^T transposed in registers (movmatrix)
// A lane keeps the running maximum and sum of heads 2c, 2c+1 (c = lane % 4).
//   o[t][0..3]: dim f8_dim(t, r) (heads 2c, 2c+1), that dim + 1 (heads 2c, 2c+1)
template <int D, int CF>
__device__ __forceinline__ void f8_chunk(const uint8_t* kt, const uint8_t* vt, int nv, const QFragSmem& qa,
                                         float scale_log2, int lane, int warp, float (&m_run)[2], float (&l_run)[2],
                                         float (&o)[D / 16][4]) {
  const int r = lane >> 2, c = lane & 3;
  const int tw = warp * 16;
  // A row's start (the 1024-byte aligned tile base plus row * D) has bits
  // 0..6 (128-byte rows) or 0..5 (64-byte rows) clear, so the swizzled address
  // of 16-byte chunk kk is (row start | swizzle key << 4 | byte) ^ (kk << 4).
  const uint32_t kts = smem_u32(kt);
  uint32_t rb[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int row = tw + h * 8 + r;
    const uint32_t key = D == 128 ? static_cast<uint32_t>(row & 7) : static_cast<uint32_t>((row >> 1) & 3);
    rb[h] = (kts + static_cast<uint32_t>(row * D)) | (key << 4) | static_cast<uint32_t>(4 * c);
  }
  float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint2 qq = qa(kk);
    uint32_t w0, w1;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(w0) : "r"(rb[0] ^ static_cast<uint32_t>(kk << 4)));
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(w1) : "r"(rb[1] ^ static_cast<uint32_t>(kk << 4)));
    uint32_t k00, k01, k10, k11;
    widen4<CF>(w0, k00, k01);  // token r: dims (4c, 4c+1), (4c+2, 4c+3) of the k-step
    widen4<CF>(w1, k10, k11);  // token r + 8
    mma16x8_f16(kk & 1 ? s1 : s0, k00, k10, k01, k11, qq.x, qq.y);
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
  // units): weights stay <= 2^8 (f16 holds them) and O is rarely rescaled
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
  // P^T as B fragments (K 16 tokens x N 8 heads), f16
  const uint32_t pb0 = movmatrix_t(pack_f16(pr[0], pr[1]));  // tokens 2c, 2c+1
  const uint32_t pb1 = movmatrix_t(pack_f16(pr[2], pr[3]));  // tokens 8+2c, 9+2c

  constexpr int W = D == 128 ? 4 : 2;  // 32-bit words of V per token this thread reads
  const int col = f8_dim<D>(0, r);
  const int t00 = tw + 2 * c, t10 = tw + 8 + 2 * c;
  const uint8_t* pa_ = vt + f8_off<D>(t00, col);
  const uint8_t* pb_ = vt + f8_off<D>(t00 + 1, col);
  const uint8_t* pc_ = vt + f8_off<D>(t10, col);
  const uint8_t* pd_ = vt + f8_off<D>(t10 + 1, col);
  const bool ragged = nv < 16;  // warp-uniform
#pragma unroll
  for (int w = 0; w < W; ++w) {
    // (token a byte k, token b byte k) pairs: bytes 0,1 then 2,3 of each word
    const uint32_t xa = *reinterpret_cast<const uint32_t*>(pa_ + 4 * w);
    const uint32_t xb = *reinterpret_cast<const uint32_t*>(pb_ + 4 * w);
    const uint32_t xc = *reinterpret_cast<const uint32_t*>(pc_ + 4 * w);
    const uint32_t xd = *reinterpret_cast<const uint32_t*>(pd_ + 4 * w);
    uint32_t b[8];
    widen4<CF>(__byte_perm(xa, xb, 0x5140), b[0], b[1]);  // dims col+4w, col+4w+1 of tokens 2c, 2c+1
    widen4<CF>(__byte_perm(xa, xb, 0x7362), b[2], b[3]);  // dims col+4w+2, col+4w+3
    widen4<CF>(__byte_perm(xc, xd, 0x5140), b[4], b[5]);  // the same of tokens 8+2c, 9+2c
    widen4<CF>(__byte_perm(xc, xd, 0x7362), b[6], b[7]);
    if (ragged) {
      // tokens past the valid ones: their V bytes may be NaN codes
      const uint32_t m0 = (2 * c < nv ? 0x0000ffffu : 0u) | (2 * c + 1 < nv ? 0xffff0000u : 0u);
      const uint32_t m1 = (2 * c + 8 < nv ? 0x0000ffffu : 0u) | (2 * c + 9 < nv ? 0xffff0000u : 0u);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        b[k] &= m0;
        b[4 + k] &= m1;
      }
    }
    // m-tile 2w: rows r, r+8 = dims col+4w, col+4w+1; m-tile 2w+1: col+4w+2, col+4w+3
    mma16x8_f16(o[2 * w], b[0], b[1], b[4], b[5], pb0, pb1);
    mma16x8_f16(o[2 * w + 1], b[2], b[3], b[6], b[7], pb0, pb1);
  }
}

// One CTA per work item (kv head, sequence, partition); grid (Hkv, B, parts),
// partition-major. Warp 4 streams the item's K/V tiles; warps 0-3 each take
// 16 tokens of every 64-token stage; the warps' states are merged through
// shared memory at the end.
template <int D, int G, int CF>
__global__ void PA_F8_LAUNCH_BOUNDS(F8Cfg<D>::kThreads) decode_f8_kernel(const __grid_constant__ CUtensorMap tmk,
                                                                       const __grid_constant__ CUtensorMap tmv,
                                                                       const DecodeArgs a) {
  using Cfg = F8Cfg<D>;
  constexpr int NW = Cfg::kConsumerWarps, C = Cfg::kChunk, S = Cfg::kStages;
  static_assert(G <= 8, "query heads of one group must fit in the MMA's 8 columns");
  static_assert(NW * G * (D + 2) * 4 <= S * Cfg::kStageBytes, "merge buffer must fit in the stage ring");

  extern __shared__ uint8_t smem_raw[];
  __shared__ PipeSmem<S> ps;
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - sraw);

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
  using Code = typename std::conditional<CF == kCodeS8, int8_t, __nv_fp8_e4m3>::type;
  const bool do_append = a.slot_mapping && pt.last;
  AppendRow<Code, D> ar;
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
    const uint32_t box_bytes = static_cast<uint32_t>(a.bs) * D;
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
        tma_load_2d(kdst, &tmk, 0, y, &ps.full[st], pol);
        tma_load_2d(kdst + Cfg::kTileBytes, &tmv, 0, y, &ps.full[st], pol);
      }
      if (do_append) ar.after_chunk(a, i, nchunks, lane);
    });
  } else {
    // q of head r as the f16 B fragments of f8_chunk's k-steps: dims
    // (16kk + 4c, +1) and (16kk + 4c + 2, +3); heads >= G zero
    struct {
      uint32_t v[D / 16][2];
    } qa;
    const __nv_bfloat16* qrow =
        static_cast<const __nv_bfloat16*>(a.q) + (static_cast<int64_t>(s) * a.hq + hq0 + (r < G ? r : 0)) * D;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      if (r < G) {
        const uint2 w = __ldg(reinterpret_cast<const uint2*>(qrow + kk * 16 + 4 * c));
        qa.v[kk][0] = pack_f16(bf16lo(w.x), bf16hi(w.x));
        qa.v[kk][1] = pack_f16(bf16lo(w.y), bf16hi(w.y));
      } else {
        qa.v[kk][0] = qa.v[kk][1] = 0u;
      }
    }
    // every consumer warp has the same fragments: warp 0 parks them in shared memory
    uint2* qsm = reinterpret_cast<uint2*>(sgen + S * Cfg::kStageBytes);
    if (warp == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) qsm[kk * 32 + lane] = make_uint2(qa.v[kk][0], qa.v[kk][1]);
    }
    consumer_bar();
    const QFragSmem qf{qsm, lane};
    for (int i = 0; i < nchunks; ++i) {
      const int st = i % S;
      if (!pipe_wait(&ps.full[st], (i / S) & 1, &ps.abort_flag)) break;
      const int nv = min(16, min(C, pt.ntok - i * C) - warp * 16);  // warp-uniform
      if (nv > 0) {
        const uint8_t* kt = sgen + st * Cfg::kStageBytes;
        f8_chunk<D, CF>(kt, kt + Cfg::kTileBytes, nv, qf, a.scale_log2, lane, warp, m_run, l_run, o);
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
        wacc[(warp * G + h) * D + f8_dim<D>(t, r)] = o[t][j] * a.v_scale;
        wacc[(warp * G + h) * D + f8_dim<D>(t, r) + 1] = o[t][2 + j] * a.v_scale;
      }
    }
  }
  __syncthreads();
  merge_warps_and_store<G, D, NW>(a, wm, wl, wacc, s, p, hq0, pt.nparts, pt.npre, tid, Cfg::kThreads);
}

}  // namespace pa
