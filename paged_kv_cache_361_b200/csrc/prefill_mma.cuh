// Paged prefill attention (causal) on the tensor cores.
//
// P2 = "PagedAttention：操作系统级 KV 缓存虚拟内存管理".
//   §3.2.1  prefill: the prompt's tokens are processed together and their K, V
//           written into the sequence's blocks (pa_reshape_and_cache); here
//           each new token attends, causally, to every earlier position of its
//           sequence through the block table (§2.3) with out =
//           softmax(scale * q K^T) V (§1.1). A chunk of n new tokens of a
//           sequence of length L sits at positions L-n .. L-1 (chunked prefill).
//
// B200 design: CTA = (kv head g, query tile, sequence). A tile is 64 MMA rows,
// row r = (token tok0 + r / G, query head g*G + r % G), so all G heads sharing
// a kv head ride in one M dimension and every K/V tile read serves 64 rows.
// Warp 4 is the TMA producer (the decode pipeline: swizzled [bs x 64] boxes of
// K and V, 64 keys per stage, keys 0 .. the tile's last position); warps 0-3
// each own 16 rows and run S = Q K^T and O += P V as full m16n8k16 bf16 MMAs,
// with P split into a bf16 high part and remainder. The causal mask is applied
// per row; a warp skips chunks that lie entirely past its rows' positions.
// Tiles are dispatched last-first (the longest key ranges start first).
//
// 8-bit cache (CF = kCodeE4M3 or kCodeS8; cascade mode only): the producer
// copies [bs x D] byte boxes of codes into a staging slot of the stage; the
// four consumer warps widen the chunk to f16 tiles in the stage (thread = row,
// half of its dims; rows past the last key as zeros), meet on an mbarrier, and
// run the same MMAs in f16 (q rounded to f16, P as one f16 operand; P3 "PagedAttention
// 和 vLLM", the section on its future: a code c stands for value(c) * scale).
// The K scale is folded into the score scale, the V scale into the partials.
#pragma once

#include "decode_f8.cuh"
#include "decode_mma.cuh"

namespace pa {

struct PrefillArgs {
  const void* q;          // prefill: [T][hq][D] new tokens; cascade: [num_seqs][hq][D] decode queries (bf16)
  const int32_t* cu_q;    // [num_seqs + 1] prefix sums of new-token counts (prefill)
  const int32_t* tables;  // [num_seqs][max_blocks]
  const int32_t* lens;    // [num_seqs] context length including the new tokens (prefill)
  float* out;             // [T][hq][D] (prefill)
  int64_t num_blocks;
  int32_t num_seqs, hq, hkv, bs, max_blocks, max_ctx, ntiles;
  float scale_log2;
  float v_scale;  // e4m3 cache: multiplies O (1 for bf16)
  // cascade (shared-prefix) mode: group j = members[offs[j] .. offs[j+1]) shares
  // its first prefix_tokens[j] tokens; CTA (g, p, j) writes the partial of
  // prefix partition p for every member row into slot max_parts + p.
  const int32_t* group_offs;
  const int32_t* group_members;
  const int32_t* group_prefix;
  int32_t prefix_part_tokens, max_parts, parts_stride;
  float* ws_ml;
  float* ws_o;
};

// d += A(16x16) * B(16x8), all 16 rows live.
__device__ __forceinline__ void mma16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                      uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// d += A(16x16) * B(16x8), f16 operands, all 16 rows live.
__device__ __forceinline__ void mma16_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Shared memory of prefill_mma_kernel: the stage ring, plus per stage a
// staging slot of K and V codes for an 8-bit cache.
template <int D, int CF>
constexpr int prefill_mma_smem_bytes() {
  return MmaCfg<D>::kSmemBytes + (CF != 0 ? MmaCfg<D>::kStages * 2 * MmaCfg<D>::kChunk * D : 0);
}

// CASCADE = false: prefill (rows = new tokens x heads, causal).
// CASCADE = true: shared-prefix decode (rows = group members x heads, every
// row sees the whole prefix partition; partial results, not rows, are stored).
#ifndef PA_PMMA_MAXNREG
#define PA_PMMA_MAXNREG 168
#endif
template <int D, int G, bool CASCADE, int CF = 0>
__global__ void __maxnreg__(PA_PMMA_MAXNREG) prefill_mma_kernel(const __grid_constant__ CUtensorMap tmk,
                                                                         const __grid_constant__ CUtensorMap tmv,
                                                                         const PrefillArgs a) {
  using Cfg = MmaCfg<D>;
  constexpr int NW = Cfg::kConsumerWarps, C = Cfg::kChunk, S = Cfg::kStages, NT = D / 8;
  constexpr int TT = 64 / G;  // tokens per tile
  static_assert(CF == 0 || CASCADE, "8-bit codes in cascade mode only (every warp visits every chunk)");
  static_assert(NW * 32 == 2 * C, "one (row, half) of the chunk per consumer thread");
  constexpr int kCodeTileBytes = C * D, kCodeStageBytes = 2 * kCodeTileBytes;

  extern __shared__ uint8_t smem_raw[];
  __shared__ PipeSmem<S> ps;
  __shared__ uint64_t conv_bar[CF != 0 ? S : 1];  // 8-bit: the consumer warps have widened stage st
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - smem_u32(smem_raw));
  const uint32_t cs0 = sbase + S * Cfg::kStageBytes;  // 8-bit: code staging slots

  const int g = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // cascade: the suffix pass, launched as this grid's programmatic dependent,
  // may start now; it waits for this whole grid before it reads the partials
  if (CASCADE) pdl_launch_dependents();

  // key range [k_begin, kend) of this CTA and the mapping of its 64 rows
  int32_t k_begin = 0, kend = 0, base = 0, tok0 = 0, n = 0, q0 = 0, moff = 0, msz = 0;
  int64_t table_row;
  if (CASCADE) {
    const int j = blockIdx.z, p = blockIdx.y;
    moff = __ldg(a.group_offs + j);
    msz = __ldg(a.group_offs + j + 1) - moff;
    const int32_t lp = __ldg(a.group_prefix + j);
    k_begin = p * a.prefix_part_tokens;
    if (msz <= 0 || msz > TT || k_begin >= lp) return;
    kend = min(k_begin + a.prefix_part_tokens, lp);
    table_row = static_cast<int64_t>(__ldg(a.group_members + moff)) * a.max_blocks;
  } else {
    const int s = blockIdx.z;
    const int tile = a.ntiles - 1 - static_cast<int>(blockIdx.y);
    q0 = __ldg(a.cu_q + s);
    n = __ldg(a.cu_q + s + 1) - q0;
    int32_t L = __ldg(a.lens + s);
    if (L < 0 || L > a.max_ctx || n < 0 || n > L) {
      if (tid == 0 && g == 0 && tile == 0) record_error(PA_ERR_DEVICE_BOUNDS, L);
      L = L < 0 ? 0 : (L > a.max_ctx ? a.max_ctx : L);
      n = n < 0 ? 0 : (n > L ? L : n);
    }
    tok0 = tile * TT;
    if (tok0 >= n) return;
    const int32_t tok_end = min(tok0 + TT, n);
    base = L - n;             // position of new token 0
    kend = base + tok_end;    // keys 0 .. kend-1 are needed
    table_row = static_cast<int64_t>(s) * a.max_blocks;
  }
  const int nchunks = (kend - k_begin + C - 1) / C;

  if (tid == 0) {
    if constexpr (CF != 0)
      for (int i = 0; i < S; ++i) mbar_init(&conv_bar[i], NW);
    pipe_init<S>(ps, NW);
  }
  __syncthreads();

  if (CF != 0 && warp == NW) {
    const uint32_t box_bytes = static_cast<uint32_t>(a.bs) * D;
    const uint64_t pol = l2_evict_last_policy();
    pipe_produce<S>(ps, nchunks, [&](int i, int st) {
      const int32_t c0 = k_begin + i * C;
      const int32_t nb = (min(C, kend - c0) + a.bs - 1) / a.bs;  // <= 8 (bs >= 8)
      int32_t blk = -1;
      bool ok = false;
      if (lane < nb) {
        blk = __ldg(a.tables + table_row + c0 / a.bs + lane);
        ok = blk >= 0 && blk < a.num_blocks;
        if (!ok) record_error(PA_ERR_DEVICE_BOUNDS, blk);
      }
      const unsigned okmask = __ballot_sync(0xffffffffu, ok);
      if (lane == 0) mbar_arrive_expect_tx(&ps.full[st], 2u * __popc(okmask) * box_bytes);
      __syncwarp();
      if (ok) {
        const int32_t y = (blk * a.hkv + g) * a.bs;
        const uint32_t dst = cs0 + st * kCodeStageBytes + lane * box_bytes;
        tma_load_2d(dst, &tmk, 0, y, &ps.full[st], pol);
        tma_load_2d(dst + kCodeTileBytes, &tmv, 0, y, &ps.full[st], pol);
      }
    });
    return;
  }
  if (warp == NW) {
    const uint32_t box_bytes = static_cast<uint32_t>(a.bs) * D * 2u;  // one (block, head) tile of K or V
    const uint64_t pol = l2_evict_last_policy();  // later tiles of this sequence read the same keys
    pipe_produce<S>(ps, nchunks, [&](int i, int st) {
      const int32_t c0 = k_begin + i * C;
      const int32_t nb = (min(C, kend - c0) + a.bs - 1) / a.bs;  // <= 8 (bs >= 8)
      int32_t blk = -1;
      bool ok = false;
      if (lane < nb) {
        blk = __ldg(a.tables + table_row + c0 / a.bs + lane);
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
    });
    return;
  }

  // ---- consumers: warp w owns tile rows [16w, 16w+16); this lane rows ra, rb = ra + 8 ----
  const int c = lane & 3;
  const int ra = warp * 16 + (lane >> 2), rb = ra + 8;
  bool va, vb;
  int pa_, pb_, wmax;
  int64_t qrow_a, qrow_b;  // q row (and output row) of each
  if (CASCADE) {
    va = ra / G < msz;
    vb = rb / G < msz;
    pa_ = va ? kend - 1 : -1;
    pb_ = vb ? kend - 1 : -1;
    wmax = kend - 1;
    const int sa = va ? __ldg(a.group_members + moff + ra / G) : 0;
    const int sb = vb ? __ldg(a.group_members + moff + rb / G) : 0;
    qrow_a = static_cast<int64_t>(sa) * a.hq + g * G + ra % G;
    qrow_b = static_cast<int64_t>(sb) * a.hq + g * G + rb % G;
  } else {
    const int ta = tok0 + ra / G, tb = tok0 + rb / G;
    va = ta < n;
    vb = tb < n;
    pa_ = va ? base + ta : -1;  // last key each row may see
    pb_ = vb ? base + tb : -1;
    wmax = base + min(tok0 + (warp * 16 + 15) / G, n - 1);  // last key any row of this warp sees
    qrow_a = (static_cast<int64_t>(q0) + (va ? ta : 0)) * a.hq + g * G + ra % G;
    qrow_b = (static_cast<int64_t>(q0) + (vb ? tb : 0)) * a.hq + g * G + rb % G;
  }
  const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(a.q);
  const uint32_t* qra = reinterpret_cast<const uint32_t*>(qb + qrow_a * D);
  const uint32_t* qrb = reinterpret_cast<const uint32_t*>(qb + qrow_b * D);
  uint32_t qa[D / 16][4];
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    qa[kk][0] = va ? __ldg(qra + kk * 8 + c) : 0u;
    qa[kk][1] = vb ? __ldg(qrb + kk * 8 + c) : 0u;
    qa[kk][2] = va ? __ldg(qra + kk * 8 + 4 + c) : 0u;
    qa[kk][3] = vb ? __ldg(qrb + kk * 8 + 4 + c) : 0u;
    if constexpr (CF != 0)
#pragma unroll
      for (int e = 0; e < 4; ++e) qa[kk][e] = pack_f16(bf16lo(qa[kk][e]), bf16hi(qa[kk][e]));
  }
  float o[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float ma = -INFINITY, mb = -INFINITY, la = 0.f, lb = 0.f;

  const int mk = lane >> 3, ik = lane & 7;
  // address of row t, dims d0 .. d0+7 of a stage tile: block-major as the TMA
  // writes it over a bf16 cache (block t / bs at t / bs * bs * D * 2 bytes,
  // 64-element half at half * bs * 128, row at (t % bs) * 128), half-major as
  // the converter writes it over an 8-bit cache; 128-byte swizzle phase t & 7
  auto tile_addr = [&](uint32_t base, int t, int d0) -> uint32_t {
    const uint32_t swz = static_cast<uint32_t>((((d0 & 63) >> 3) ^ (t & 7)) << 4);
    if constexpr (CF != 0)
      return base + (d0 >> 6) * Cfg::kHalfBytes + t * 128 + swz;
    else
      return base + (t + (t & ~(a.bs - 1)) * (Cfg::kHalves - 1)) * 128 + (d0 >> 6) * a.bs * 128 + swz;
  };
  for (int i = 0; i < nchunks; ++i) {
    const int st = i % S;
    if (!pipe_wait(&ps.full[st], (i / S) & 1, &ps.abort_flag)) break;
    const int k0 = k_begin + i * C;
    if constexpr (CF != 0) {
      // widen the chunk into the stage's f16 tiles; every warp reads all of it
      const int row = tid >> 1, half = tid & 1;
      const uint8_t* src = sgen + (cs0 - sbase) + st * kCodeStageBytes;
      uint8_t* dst = sgen + st * Cfg::kStageBytes;
      widen_row_half<D, CF, Cfg::kHalfBytes>(src, dst, row, half, k0 + row < kend);
      widen_row_half<D, CF, Cfg::kHalfBytes>(src + kCodeTileBytes, dst + Cfg::kTileBytes, row, half,
                                             k0 + row < kend);
      __syncwarp();
      if (lane == 0) mbar_arrive(&conv_bar[st]);
      if (!pipe_wait(&conv_bar[st], (i / S) & 1, &ps.abort_flag)) break;
    }
    if (k0 <= wmax) {
      const uint32_t kst = sbase + st * Cfg::kStageBytes;
      const uint32_t vst = kst + Cfg::kTileBytes;
      float sacc[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int d0 = kk * 16 + (mk & 1) * 8;
#pragma unroll
        for (int kg = 0; kg < 4; ++kg) {
          const int tk = kg * 16 + (mk >> 1) * 8 + ik;
          const uint32_t addr = tile_addr(kst, tk, d0);
          uint32_t b00, b01, b10, b11;
          ldsm_x4(addr, b00, b01, b10, b11);
          if constexpr (CF != 0) {
            mma16_f16(sacc[2 * kg], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b00, b01);
            mma16_f16(sacc[2 * kg + 1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b10, b11);
          } else {
            mma16(sacc[2 * kg], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b00, b01);
            mma16(sacc[2 * kg + 1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b10, b11);
          }
        }
      }
      // causal mask and online softmax for rows ra (c0, c1) and rb (c2, c3)
      float mla = -INFINITY, mlb = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int key = k0 + nt * 8 + 2 * c + j;
          sacc[nt][j] = key <= pa_ ? sacc[nt][j] * a.scale_log2 : -INFINITY;
          sacc[nt][2 + j] = key <= pb_ ? sacc[nt][2 + j] * a.scale_log2 : -INFINITY;
          mla = fmaxf(mla, sacc[nt][j]);
          mlb = fmaxf(mlb, sacc[nt][2 + j]);
        }
      mla = fmaxf(mla, __shfl_xor_sync(0xffffffffu, mla, 1));
      mla = fmaxf(mla, __shfl_xor_sync(0xffffffffu, mla, 2));
      mlb = fmaxf(mlb, __shfl_xor_sync(0xffffffffu, mlb, 1));
      mlb = fmaxf(mlb, __shfl_xor_sync(0xffffffffu, mlb, 2));
      const float na = fmaxf(ma, mla), nb = fmaxf(mb, mlb);
      // a row with nothing visible yet keeps m = -inf; its weights are 0
      const float alpha_a = na == -INFINITY ? 1.f : exp2f(ma - na);
      const float alpha_b = nb == -INFINITY ? 1.f : exp2f(mb - nb);
      float suma = 0.f, sumb = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          sacc[nt][j] = na == -INFINITY ? 0.f : exp2f(sacc[nt][j] - na);
          sacc[nt][2 + j] = nb == -INFINITY ? 0.f : exp2f(sacc[nt][2 + j] - nb);
          suma += sacc[nt][j];
          sumb += sacc[nt][2 + j];
        }
      ma = na;
      mb = nb;
      la = la * alpha_a + suma;
      lb = lb * alpha_b + sumb;
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        o[j][0] *= alpha_a;
        o[j][1] *= alpha_a;
        o[j][2] *= alpha_b;
        o[j][3] *= alpha_b;
      }
      // O += P V, 16 keys (n-tiles 2kg, 2kg+1) per k-step; V rows past kend are zeroed
      const int nvk = min(C, kend - k0);
#pragma unroll
      for (int kg = 0; kg < 4; ++kg) {
        uint32_t h0, l0, h1, l1, h2, l2, h3, l3;
        if constexpr (CF != 0) {  // weights <= 1 as f16, one MMA
          h0 = pack_f16(sacc[2 * kg][0], sacc[2 * kg][1]);
          h1 = pack_f16(sacc[2 * kg][2], sacc[2 * kg][3]);
          h2 = pack_f16(sacc[2 * kg + 1][0], sacc[2 * kg + 1][1]);
          h3 = pack_f16(sacc[2 * kg + 1][2], sacc[2 * kg + 1][3]);
          l0 = l1 = l2 = l3 = 0u;
        } else {
          split_pair(sacc[2 * kg][0], sacc[2 * kg][1], h0, l0);          // row ra, keys 2c, 2c+1
          split_pair(sacc[2 * kg][2], sacc[2 * kg][3], h1, l1);          // row rb
          split_pair(sacc[2 * kg + 1][0], sacc[2 * kg + 1][1], h2, l2);  // row ra, keys +8
          split_pair(sacc[2 * kg + 1][2], sacc[2 * kg + 1][3], h3, l3);  // row rb, keys +8
        }
        const int kb = kg * 16;
        uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
        if (kb + 16 > nvk) {
          mlo = (kb + 2 * c < nvk ? 0x0000ffffu : 0u) | (kb + 2 * c + 1 < nvk ? 0xffff0000u : 0u);
          mhi = (kb + 2 * c + 8 < nvk ? 0x0000ffffu : 0u) | (kb + 2 * c + 9 < nvk ? 0xffff0000u : 0u);
        }
        const int tv = kb + (mk & 1) * 8 + ik;
#pragma unroll
        for (int dg = 0; dg < D / 16; ++dg) {
          const int d0 = dg * 16 + (mk >> 1) * 8;
          const uint32_t addr = tile_addr(vst, tv, d0);
          uint32_t v0, v1, v2, v3;
          ldsm_x4_t(addr, v0, v1, v2, v3);
          v0 &= mlo;
          v1 &= mhi;
          v2 &= mlo;
          v3 &= mhi;
          if constexpr (CF != 0) {
            mma16_f16(o[2 * dg], h0, h1, h2, h3, v0, v1);
            mma16_f16(o[2 * dg + 1], h0, h1, h2, h3, v2, v3);
          } else {
            mma16(o[2 * dg], h0, h1, h2, h3, v0, v1);
            mma16(o[2 * dg], l0, l1, l2, l3, v0, v1);
            mma16(o[2 * dg + 1], h0, h1, h2, h3, v2, v3);
            mma16(o[2 * dg + 1], l0, l1, l2, l3, v2, v3);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&ps.empty[st]);
  }
  if (ps.abort_flag) return;

  la += __shfl_xor_sync(0xffffffffu, la, 1);
  la += __shfl_xor_sync(0xffffffffu, la, 2);
  lb += __shfl_xor_sync(0xffffffffu, lb, 1);
  lb += __shfl_xor_sync(0xffffffffu, lb, 2);
  if (CASCADE) {
    // partials of prefix partition blockIdx.y: unnormalised o (times the V
    // scale of an 8-bit cache, 1 otherwise), (m, l)
    const int slot = a.max_parts + static_cast<int>(blockIdx.y);
    const float vs = a.v_scale;
    if (va) {
      const int64_t prow = qrow_a * a.parts_stride + slot;
      float* dst = a.ws_o + prow * D + 2 * c;
#pragma unroll
      for (int j = 0; j < NT; ++j)
        *reinterpret_cast<float2*>(dst + j * 8) = make_float2(o[j][0] * vs, o[j][1] * vs);
      if (c == 0) *reinterpret_cast<float2*>(a.ws_ml + prow * 2) = make_float2(ma, la);
    }
    if (vb) {
      const int64_t prow = qrow_b * a.parts_stride + slot;
      float* dst = a.ws_o + prow * D + 2 * c;
#pragma unroll
      for (int j = 0; j < NT; ++j)
        *reinterpret_cast<float2*>(dst + j * 8) = make_float2(o[j][2] * vs, o[j][3] * vs);
      if (c == 0) *reinterpret_cast<float2*>(a.ws_ml + prow * 2) = make_float2(mb, lb);
    }
    return;
  }
  if (va) {
    const float inv = 1.f / la;
    float* dst = a.out + qrow_a * D + 2 * c;
#pragma unroll
    for (int j = 0; j < NT; ++j) *reinterpret_cast<float2*>(dst + j * 8) = make_float2(o[j][0] * inv, o[j][1] * inv);
  }
  if (vb) {
    const float inv = 1.f / lb;
    float* dst = a.out + qrow_b * D + 2 * c;
#pragma unroll
    for (int j = 0; j < NT; ++j) *reinterpret_cast<float2*>(dst + j * 8) = make_float2(o[j][2] * inv, o[j][3] * inv);
  }
}

}  // namespace pa
