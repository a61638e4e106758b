// Paged prefill attention (causal) on the 5th-generation tensor cores:
// tcgen05.mma with the accumulators in tensor memory (TMEM).
//
// P2 = "PagedAttention：操作系统级 KV 缓存虚拟内存管理".
//   §3.2.1  prefill: the prompt's tokens are processed together and their K, V
//           written into the sequence's blocks (pa_reshape_and_cache); each
//           new token attends, causally, to every earlier position of its
//           sequence through the block table (§2.3) with
//           out = softmax(scale * q K^T) V (§1.1). A chunk of n new tokens of a
//           sequence of length L sits at positions L-n .. L-1.
//
// CTA = (kv head g, query tile, sequence); a tile is 128 rows (the MMA M),
// row r = (token tok0 + r / G, query head g*G + r % G), so the G heads sharing
// a kv head read every K/V tile once. Warps:
//   warp 4     TMA producer: swizzled [bs x 64] boxes of K, 64 keys per stage;
//              over a bf16 cache a second producer warp (after the converter
//              warps) copies the stage's V, so that K and V are released
//              separately: K once both tiles' S = Q K^T has read it, V after
//              their P V. (Over an 8-bit cache one producer copies both.)
//   warp 5     allocates TMEM and walks the MMA schedule; one lane chosen
//              by elect.sync issues every MMA:
//                S_j = Q K_j^T        (M 128, N 64, K = D; A and B in shared
//                                      memory, K-major) into TMEM buffer j % 2
//                O  += P_j V_j        (M 128, N = D, K 64; A = P from TMEM,
//                                      B = V in shared memory, N-major)
//              S_{j+1} is issued before O += P_j V_j so the tensor core works
//              while the softmax warps handle chunk j. Completions reach the
//              other warps through tcgen05.commit on mbarriers.
//   warps 0-3  one thread per row (TMEM lane): per chunk read S from TMEM,
//              mask causally, keep the running maximum m and sum l in base
//              2, write P back into the S buffer as f16 (11 significant
//              bits; weights are at most 2^8); at the end read O, divide by
//              l and store it fp32 through shared memory (the CTA's last
//              tile by TMA stores from the freed K/V stages). Q of a tile
//              whose rows all lie in the sequence arrives by TMA (bf16
//              cache); otherwise these threads load it row by row.
//   warps +2..+5  converter: a kind::f16 MMA takes A and B of one type, so
//              with P in f16 the V operand must be f16 too. The converter
//              rewrites each stage's V tile in place, bf16 -> f16 (exact for
//              normal f16 values, |v| <= 65504; values below 2^-14 keep their
//              f16 subnormal bits, an absolute change below 2^-25), and writes
//              rows past the stream's last key as zeros (their bytes may be
//              padding or NaN), then releases the stage's V to the MMA warp.
//              S = Q K^T stays bf16 x bf16 (Q and K straight from the cache).
// The running maximum is moved (and O rescaled in TMEM) only when a row's
// maximum grows by more than 8 in log2 units, so weights stay below 2^8 and
// most chunks never touch O; the result is the same softmax.
//
// 8-bit cache (CF: e4m3 or int8 codes). P3 = "PagedAttention 和 vLLM", the
// section on its future: paged KV storage combined with quantisation, a code c
// standing for value(c) * scale with one scale per tensor. The keys and values
// are widened to f16 (cvt e4m3x2 -> f16x2, or the int8 byte-permute widening;
// both exact) by the converter role: the producer copies [bs x D] byte boxes
// of codes (128-byte swizzle at D 128, 64-byte at D 64) into a small staging
// ring; the converter writes each chunk as f16 K and V tiles in the swizzled
// layout the bf16 path gets from the TMA, with rows past the stream's last key
// written as zeros (their bytes may be anything, a NaN code included).
// Q is rounded to f16 by the softmax warps as they stage it (exact for
// 2^-17 <= |q| <= 65504). The K scale is folded into the score scale; the V
// scale multiplies O in the final division.
#pragma once

#include "decode_f8.cuh"
#include "prefill_mma.cuh"
#include "tcgen05.cuh"

namespace pa {

// Build-time knob: K/V stages of the bf16 path (64 keys each; 5 still fits
// beside two Q tiles at head_dim 128).
#ifndef PA_TC_STAGES
#define PA_TC_STAGES 4
#endif


template <int D, int TILES, bool F8 = false>
struct TcCfg {
  static constexpr int kRows = 128;                        // query rows per tile (MMA M)
  static constexpr int kChunk = 64;                        // keys per stage
  static constexpr int kHalves = D / 64;                   // 128-byte column boxes per row
  static constexpr int kHalfBytes = kChunk * 128;          // one box column of K or V in a stage
  static constexpr int kTileBytes = kHalves * kHalfBytes;  // K (or V) of one stage (16-bit elements)
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStages = F8 && TILES > 1 ? 3 : PA_TC_STAGES;
  static constexpr int kCodeTileBytes = kChunk * D;        // 8-bit K (or V) codes of one staging slot
  static constexpr int kCodeStageBytes = 2 * kCodeTileBytes;
  static constexpr int kCodeStages = F8 ? (TILES > 1 ? 2 : 3) : 0;
  static constexpr int kQHalfBytes = kRows * 128;
  static constexpr int kQTileBytes = kHalves * kQHalfBytes;
  static constexpr int kQBytes = TILES * kQTileBytes;
  static constexpr int kSmemBytes = 1024 + kQBytes + kStages * kStageBytes + kCodeStages * kCodeStageBytes;
  static constexpr int kSoftmaxWarps = 4 * TILES;          // one warpgroup per tile
  static constexpr int kProducerWarp = kSoftmaxWarps;
  static constexpr int kMmaWarp = kSoftmaxWarps + 1;
  static constexpr int kConvWarp0 = kSoftmaxWarps + 2;
  static constexpr int kConvWarps = 4;
  // bf16: a second producer warp streams V (K and V of a stage are released
  // separately: K once both tiles' S has read it, V after their P V)
  static constexpr int kVProducerWarp = kConvWarp0 + kConvWarps;
  static constexpr int kThreads = 32 * (kSoftmaxWarps + 2 + kConvWarps + (F8 ? 0 : 1));
  // per tile: O (D columns), then two S/P buffers of kChunk columns
  static constexpr uint32_t kTileCols = D + 2 * kChunk;
  static constexpr uint32_t kTmemCols = TILES * kTileCols <= 256 ? 256 : 512;
  static_assert(TILES * kTileCols <= kTmemCols, "TMEM columns");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

// One row of a stage's V tile (64 keys x D, bf16, as the TMA wrote it:
// [rows x 64] box columns of 128-byte rows with the 128-byte swizzle,
// kHalfBytes apart), rewritten in place as f16: the box column `half` at
// D 128, or the half `half` of the single 128-byte row at D 64. live = false
// writes zeros. At D 128 the two box columns of a row are handled by
// neighbouring lanes; half 1 walks its 16-byte chunks in rotated order so that
// the eight lanes of a shared-memory phase touch eight different chunk
// positions (at D 64 the two halves already do).
template <int D, int kHalfBytes>
__device__ __forceinline__ void v_to_f16_inplace(uint8_t* vt, int row, int half, bool live) {
  constexpr int NCH = D == 128 ? 8 : 4;  // 16-byte chunks per thread
  uint8_t* rp = vt + (D == 128 ? half * kHalfBytes : 0) + row * 128;
  uint4* ptr[NCH];
  uint4 x[NCH];
  // every load of the row's pieces first (all in flight together), then the stores
#pragma unroll
  for (int u0 = 0; u0 < NCH; ++u0) {
    const int c = D == 128 ? (half ? (u0 ^ 4) : u0) : half * 4 + u0;  // logical chunk of the 128-byte row
    ptr[u0] = reinterpret_cast<uint4*>(rp + ((c ^ (row & 7)) << 4));
    x[u0] = live ? *ptr[u0] : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int u0 = 0; u0 < NCH; ++u0)
    *ptr[u0] = make_uint4(pack_f16(bf16lo(x[u0].x), bf16hi(x[u0].x)), pack_f16(bf16lo(x[u0].y), bf16hi(x[u0].y)),
                          pack_f16(bf16lo(x[u0].z), bf16hi(x[u0].z)), pack_f16(bf16lo(x[u0].w), bf16hi(x[u0].w)));
}

// All lanes wait; the warp proceeds only if every lane saw the phase.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const bool ok = pipe_wait(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

// TMA store of one box of a 3-D map from shared memory (coordinates x, y, z),
// in this thread's bulk group; the group's reads of shared memory are awaited
// with bulk_wait_read.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int32_t x, int32_t y, int32_t z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y), "r"(z)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// TILES query tiles of one (kv head, sequence) per CTA share the K/V stream;
// tile t is processed by softmax warpgroup t.
// CF = 0: bf16 cache; kCodeE4M3 / kCodeS8: an 8-bit cache of that format.
template <int D, int G, int TILES, int CF = 0>
__global__ void __launch_bounds__(TcCfg<D, TILES, CF != 0>::kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                      const __grid_constant__ CUtensorMap tmo, const __grid_constant__ CUtensorMap tmq,
                      const PrefillArgs a) {
  constexpr bool F8 = CF != 0;
  using Cfg = TcCfg<D, TILES, F8>;
  constexpr int S = Cfg::kStages, C = Cfg::kChunk, TT = Cfg::kRows / G;
  constexpr int CS = F8 ? Cfg::kCodeStages : 1;

  extern __shared__ uint8_t smem_raw[];
  __shared__ PipeSmem<S> ps;  // 16-bit K/V stages: filled by the TMA (bf16) or the converter (F8)
  __shared__ uint64_t cfull[CS], cempty[CS];  // F8: code staging ring, producer <-> converter
  __shared__ uint64_t vready[S];              // bf16: the stage's V rewritten as f16 (converter -> MMA)
  __shared__ uint64_t vfull[S], vempty[S];    // bf16: V of a stage (ps.full / ps.empty track its K)
  __shared__ uint64_t q_full, drain;
  __shared__ uint64_t s_full[TILES][2], p_full[TILES][2], o_bar[TILES];
  __shared__ uint64_t o_last[TILES];  // one phase: tile t's last P V (and every MMA before it) complete
  __shared__ uint64_t o_staged;       // the last tile's O is in shared memory (one arrival per warp)
  __shared__ uint32_t tmem_base_sh;
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);   // generic pointer to sbase
  const uint32_t qs = sbase;                  // Q of tile t: kHalves x [128 rows x 128 B], swizzled
  const uint32_t kv0 = sbase + Cfg::kQBytes;  // stage st: K halves, then V halves
  const uint32_t cs0 = kv0 + S * Cfg::kStageBytes;  // F8 staging slot: K codes, then V codes

  // grid (kv heads, sequences, tile pairs): every sequence's last (longest) pair
  // is dispatched before any shorter one, so the last CTAs to run are the short ones
  const int g = blockIdx.x, s = blockIdx.y;
  const int pair = a.ntiles - 1 - static_cast<int>(blockIdx.z);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
    prefetch_tmap(&tmq);
    prefetch_tmap(&tmo);
  }

  const int32_t q0 = __ldg(a.cu_q + s);
  int32_t n = __ldg(a.cu_q + s + 1) - q0;
  int32_t L = __ldg(a.lens + s);
  if (L < 0 || L > a.max_ctx || n < 0 || n > L) {
    if (tid == 0 && g == 0 && pair == 0) record_error(PA_ERR_DEVICE_BOUNDS, L);
    L = L < 0 ? 0 : (L > a.max_ctx ? a.max_ctx : L);
    n = n < 0 ? 0 : (n > L ? L : n);
  }
  const int32_t base = L - n;  // position of new token 0
  const int32_t tok00 = pair * TILES * TT;
  if (tok00 >= n) return;
  // per tile: first token, key end, chunks; the stream follows the last active tile
  int ntiles_act = 0, nch[TILES];
  int32_t kend_all = 0;
#pragma unroll
  for (int t = 0; t < TILES; ++t) {
    const int32_t t0 = tok00 + t * TT;
    nch[t] = 0;
    if (t0 < n) {
      const int32_t ke = base + min(t0 + TT, n);
      nch[t] = (ke + C - 1) / C;
      kend_all = ke;
      ntiles_act = t + 1;
    }
  }
  const int nchunks = nch[ntiles_act - 1];
  const int64_t table_row = static_cast<int64_t>(s) * a.max_blocks;
  // Q of a tile whose rows all lie inside the sequence arrives by TMA (bf16:
  // the rows as they are); otherwise the softmax warps load it row by row
  // (zeros past the sequence; f16 over an 8-bit cache)
  auto q_by_tma = [&](int t) { return !F8 && t < ntiles_act && tok00 + (t + 1) * TT <= n; };
  int q_arrivals = 0, q_tma_tiles = 0;
#pragma unroll
  for (int t = 0; t < TILES; ++t) {
    if (q_by_tma(t)) ++q_tma_tiles;
    else if (t < ntiles_act) q_arrivals += 4;
  }

  if (tid == 0) {
    mbar_init(&q_full, q_arrivals + (q_tma_tiles > 0 ? 1 : 0));
    mbar_init(&drain, 1);
    mbar_init(&o_staged, 4);
#pragma unroll
    for (int t = 0; t < TILES; ++t) {
      mbar_init(&s_full[t][0], 1);
      mbar_init(&s_full[t][1], 1);
      mbar_init(&p_full[t][0], 4);
      mbar_init(&p_full[t][1], 4);
      mbar_init(&o_bar[t], 1);
      mbar_init(&o_last[t], 1);
    }
    if constexpr (F8) {
#pragma unroll
      for (int i = 0; i < S; ++i) {
        mbar_init(&ps.full[i], Cfg::kConvWarps);
        mbar_init(&ps.empty[i], 1);
      }
#pragma unroll
      for (int i = 0; i < CS; ++i) {
        mbar_init(&cfull[i], 1);
        mbar_init(&cempty[i], Cfg::kConvWarps);
      }
      ps.abort_flag = 0;
      fence_mbar_init();
    } else {
#pragma unroll
      for (int i = 0; i < S; ++i) {
        mbar_init(&vready[i], Cfg::kConvWarps);
        mbar_init(&vfull[i], 1);
        mbar_init(&vempty[i], 1);
      }
      pipe_init<S>(ps, 1);  // empty stages are released by one tcgen05.commit
    }
    if (q_tma_tiles > 0) {
      // [128 / G tokens x G heads x 64 dims] boxes, one per 64-dim half of a tile
      mbar_arrive_expect_tx(&q_full, static_cast<uint32_t>(q_tma_tiles * Cfg::kQTileBytes));
      const uint64_t pol = l2_evict_first_policy();
#pragma unroll
      for (int t = 0; t < TILES; ++t)
        if (q_by_tma(t)) {
#pragma unroll
          for (int hf = 0; hf < Cfg::kHalves; ++hf)
            tma_load_3d(sbase + t * Cfg::kQTileBytes + hf * Cfg::kQHalfBytes, &tmq, hf * 64, g * G,
                        q0 + tok00 + t * TT, &q_full, pol);
        }
    }
  }
  // the producers' first block-table window is read while the CTA sets up
  // (its ids feed the first K/V copies: one memory round trip less at the start)
  TableAhead ta;
  if (warp == Cfg::kProducerWarp || (!F8 && warp == Cfg::kVProducerWarp))
    ta.init(a.tables + table_row, 0, min(a.max_blocks, (kend_all + a.bs - 1) / a.bs), lane);
  if (warp == Cfg::kMmaWarp) {
    tc::alloc(smem_u32(&tmem_base_sh), Cfg::kTmemCols);
    tc::relinquish();
    tc::fence_before();
  }
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (F8 && warp == Cfg::kProducerWarp) {
    // ---- producer (F8): codes of chunk i into staging slot i % CS ----
    const uint32_t box_bytes = static_cast<uint32_t>(a.bs) * D;
    const uint64_t pol = l2_evict_last_policy();
    int i = 0;
    for (; i < nchunks; ++i) {
      const int cst = i % CS;
      if (i >= CS && !warp_wait(&cempty[cst], ((i / CS) - 1) & 1, &ps.abort_flag)) break;
      const int32_t c0 = i * C;
      const int32_t nb = (min(C, kend_all - c0) + a.bs - 1) / a.bs;  // <= 8 (bs >= 8)
      const int32_t blk = ta.get(c0 / a.bs, nb, lane);
      bool ok = false;
      if (lane < nb) {
        ok = blk >= 0 && blk < a.num_blocks;
        if (!ok) record_error(PA_ERR_DEVICE_BOUNDS, blk);
      }
      const unsigned okmask = __ballot_sync(0xffffffffu, ok);
      if (lane == 0) mbar_arrive_expect_tx(&cfull[cst], 2u * __popc(okmask) * box_bytes);
      __syncwarp();
      if (ok) {
        const int32_t y = (blk * a.hkv + g) * a.bs;
        const uint32_t dst = cs0 + cst * Cfg::kCodeStageBytes + lane * box_bytes;
        tma_load_2d(dst, &tmk, 0, y, &cfull[cst], pol);
        tma_load_2d(dst + Cfg::kCodeTileBytes, &tmv, 0, y, &cfull[cst], pol);
      }
    }
    if (ps.abort_flag && lane == 0)  // copies already started land before exit
      for (int j = (i > CS ? i - CS : 0); j < i; ++j) mbar_wait(&cfull[j % CS], (j / CS) & 1);
  } else if (F8 && warp >= Cfg::kConvWarp0) {
    // ---- converter (F8): thread = (row of the chunk, half of its dims) ----
    const int ct = tid - 32 * Cfg::kConvWarp0;
    const int row = ct >> 1, half = ct & 1;
    const uint8_t* cs0g = sgen + (cs0 - sbase);
    uint8_t* kv0g = sgen + Cfg::kQBytes;
    for (int i = 0; i < nchunks; ++i) {
      const int cst = i % CS, st = i % S;
      if (!warp_wait(&cfull[cst], (i / CS) & 1, &ps.abort_flag)) break;
      if (i >= S && !warp_wait(&ps.empty[st], ((i / S) - 1) & 1, &ps.abort_flag)) break;
      const bool live = i * C + row < kend_all;  // rows past the last key become zeros
      const uint8_t* src = cs0g + cst * Cfg::kCodeStageBytes;
      uint8_t* dst = kv0g + st * Cfg::kStageBytes;
      widen_row_half<D, CF, Cfg::kHalfBytes>(src, dst, row, half, live);
      widen_row_half<D, CF, Cfg::kHalfBytes>(src + Cfg::kCodeTileBytes, dst + Cfg::kTileBytes, row, half, live);
      tc::fence_proxy_async();  // generic-proxy writes -> tensor-core reads
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&ps.full[st]);
        mbar_arrive(&cempty[cst]);
      }
    }
  } else if (!F8 && warp >= Cfg::kConvWarp0 && warp < Cfg::kConvWarp0 + Cfg::kConvWarps) {
    // ---- converter (bf16): the stage's V tile, bf16 -> f16 in place; thread =
    // (row of the chunk, box column at D 128 / half of the row at D 64) ----
    const int ct = tid - 32 * Cfg::kConvWarp0;
    const int row = ct >> 1, half = ct & 1;
    uint8_t* kv0g = sgen + Cfg::kQBytes;
    for (int i = 0; i < nchunks; ++i) {
      const int st = i % S;
      if (!warp_wait(&vfull[st], (i / S) & 1, &ps.abort_flag)) break;
      const bool live = i * C + row < kend_all;  // rows past the last key become zeros
      v_to_f16_inplace<D, Cfg::kHalfBytes>(kv0g + st * Cfg::kStageBytes + Cfg::kTileBytes, row, half, live);
      tc::fence_proxy_async();  // generic-proxy writes -> tensor-core reads
      __syncwarp();
      if (lane == 0) mbar_arrive(&vready[st]);
    }
  } else if (!F8 && (warp == Cfg::kProducerWarp || warp == Cfg::kVProducerWarp)) {
    // ---- producers (bf16): K of chunk i into stage i % S (released by the S
    // MMAs) by one warp, V (released by the P V MMAs) by the other ----
    const bool is_v = warp == Cfg::kVProducerWarp;
    uint64_t* full = is_v ? vfull : ps.full;
    uint64_t* empty = is_v ? vempty : ps.empty;
    const CUtensorMap* map = is_v ? &tmv : &tmk;
    const uint32_t tile_off = is_v ? Cfg::kTileBytes : 0u;
    const uint32_t box_bytes = static_cast<uint32_t>(a.bs) * 128u;
    const uint64_t pol = l2_evict_last_policy();  // later tiles of this sequence read the same keys
    int i = 0;
    for (; i < nchunks; ++i) {
      const int st = i % S;
      if (i >= S && !warp_wait(&empty[st], ((i / S) - 1) & 1, &ps.abort_flag)) break;
      const int32_t c0 = i * C;
      const int32_t nb = (min(C, kend_all - c0) + a.bs - 1) / a.bs;  // <= 8 (bs >= 8)
      const int32_t blk = ta.get(c0 / a.bs, nb, lane);
      bool ok = false;
      if (lane < nb) {
        ok = blk >= 0 && blk < a.num_blocks;
        if (!ok && !is_v) record_error(PA_ERR_DEVICE_BOUNDS, blk);
      }
      const unsigned okmask = __ballot_sync(0xffffffffu, ok);
      if (lane == 0) mbar_arrive_expect_tx(&full[st], Cfg::kHalves * __popc(okmask) * box_bytes);
      __syncwarp();
      if (ok) {
        const int32_t y = (blk * a.hkv + g) * a.bs;
        const uint32_t dst = kv0 + st * Cfg::kStageBytes + tile_off + lane * box_bytes;
#pragma unroll
        for (int hf = 0; hf < Cfg::kHalves; ++hf) tma_load_2d(dst + hf * Cfg::kHalfBytes, map, hf * 64, y, &full[st], pol);
      }
    }
    if (ps.abort_flag && lane == 0)  // copies already started land before exit
      for (int j = (i > S ? i - S : 0); j < i; ++j) mbar_wait(&full[j % S], (j / S) & 1);
  } else if (warp == Cfg::kMmaWarp) {
    // ---- MMA issuer: S_t(j+1) for every tile, then O_t += P_t(j) V(j); the
    // whole warp walks the schedule and waits, one elected lane issues ----
    {
      constexpr uint32_t kIdS = F8 ? tc::idesc_f16(Cfg::kRows, C, false) : tc::idesc_bf16(Cfg::kRows, C, false);
      constexpr uint32_t kIdPV = tc::idesc_f16(Cfg::kRows, D, true);  // P and V as f16
      // Descriptors are built once; an operand at a byte offset from a base
      // is the base descriptor plus offset / 16 (the start-address field,
      // addresses stay below 256 KB so the field never carries over).
      const uint64_t qdesc0 = tc::smem_desc(qs, 16, 1024);
      const uint64_t kdesc0 = tc::smem_desc(kv0, 16, 1024);
      const uint64_t vdesc0 =
          tc::smem_desc(kv0 + Cfg::kTileBytes, Cfg::kHalves > 1 ? Cfg::kHalfBytes : 1024, 1024);
      auto issue_s = [&](int t, int j) {
        const uint64_t qb = qdesc0 + static_cast<uint64_t>((t * Cfg::kQTileBytes) >> 4);
        const uint64_t kb = kdesc0 + static_cast<uint64_t>(((j % S) * Cfg::kStageBytes) >> 4);
        const uint32_t dst = tmem + t * Cfg::kTileCols + D + (j & 1) * C;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // 16 dims = 32 B along the swizzled 128-byte row; 64 dims per box column
          const uint32_t offq = static_cast<uint32_t>((kk >> 2) * Cfg::kQHalfBytes + (kk & 3) * 32) >> 4;
          const uint32_t offk = static_cast<uint32_t>((kk >> 2) * Cfg::kHalfBytes + (kk & 3) * 32) >> 4;
          tc::mma_ss(dst, qb + offq, kb + offk, kIdS, kk > 0);
        }
        tc::commit(smem_u32(&s_full[t][j & 1]));
      };
      auto issue_pv = [&](int t, int j) -> bool {
        const int sb = j & 1;
        if (!warp_wait(&p_full[t][sb], (j >> 1) & 1, &ps.abort_flag)) return false;
        tc::fence_after();
        // V is N-major: 8-key groups 1024 B apart, the two 64-column halves
        // kHalfBytes apart (one half when D = 64: the offset is then unused)
        const uint64_t vb = vdesc0 + static_cast<uint64_t>(((j % S) * Cfg::kStageBytes) >> 4);
        const uint32_t to = tmem + t * Cfg::kTileCols;
        const uint32_t tp = to + D + sb * C;  // P as f16: 32 columns
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks) {
          const uint64_t bd = vb + static_cast<uint64_t>((ks * 16 * 128) >> 4);
          tc::mma_ts(to, tp + ks * 8, bd, kIdPV, j > 0 || ks > 0);
        }
        tc::commit(smem_u32(&o_bar[t]));
        if (j == nch[t] - 1) tc::commit(smem_u32(&o_last[t]));
        return true;
      };
      bool ok = warp_wait(&q_full, 0, &ps.abort_flag);
      ok = ok && warp_wait(&ps.full[0], 0, &ps.abort_flag);
      tc::fence_after();
      if (ok) {
#pragma unroll
        for (int t = 0; t < TILES; ++t)
          if (nch[t] > 0) issue_s(t, 0);
        if constexpr (!F8) tc::commit(smem_u32(&ps.empty[0]));  // K of stage 0 is read once these finish
      }
      for (int j = 0; ok && j < nchunks; ++j) {
        if (j + 1 < nchunks) {
          if (!warp_wait(&ps.full[(j + 1) % S], ((j + 1) / S) & 1, &ps.abort_flag)) {
            ok = false;
            break;
          }
          tc::fence_after();
#pragma unroll
          for (int t = 0; t < TILES; ++t)
            if (j + 1 < nch[t]) issue_s(t, j + 1);
          if constexpr (!F8) tc::commit(smem_u32(&ps.empty[(j + 1) % S]));  // K of chunk j+1 released
        }
        if constexpr (!F8) {
          // the converter has rewritten this stage's V as f16
          if (!warp_wait(&vready[j % S], (j / S) & 1, &ps.abort_flag)) {
            ok = false;
            break;
          }
          tc::fence_after();
        }
#pragma unroll
        for (int t = 0; t < TILES; ++t)
          if (ok && j < nch[t]) ok = issue_pv(t, j);
        // every tile is done with stage j (bf16: its V; 8-bit: the whole stage)
        if (ok) tc::commit(smem_u32(F8 ? &ps.empty[j % S] : &vempty[j % S]));
      }
      // every MMA the warp issued has finished before TMEM is released
      tc::commit(smem_u32(&drain));
      mbar_wait(&drain, 0);
    }
    __syncwarp();
  } else {
    // ---- softmax warpgroup t: thread = row = TMEM lane ----
    const int t = warp >> 2;
    const int r = tid & 127;
    const int32_t tok0 = tok00 + t * TT;
    const int mych = nch[t];
    if (mych > 0) {
      const int32_t tok_end = min(tok0 + TT, n);
      const int tok = tok0 + r / G;
      const bool valid = tok < n;
      const int32_t pos = base + (valid ? tok : tok_end - 1);  // last key the row sees
      const int h = r % G;
      const int64_t orow = (static_cast<int64_t>(q0) + (valid ? tok : 0)) * a.hq + g * G + h;
      if (!q_by_tma(t)) {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) + orow * D);
        uint8_t* qdst = sgen + t * Cfg::kQTileBytes;
        // every piece of the row in flight at once, then the shared-memory stores
        uint4 qv[D / 8];
#pragma unroll
        for (int c16 = 0; c16 < D / 8; ++c16) qv[c16] = valid ? __ldg(src + c16) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int c16 = 0; c16 < D / 8; ++c16) {
          uint4 v = qv[c16];
          if constexpr (F8)
            v = make_uint4(pack_f16(bf16lo(v.x), bf16hi(v.x)), pack_f16(bf16lo(v.y), bf16hi(v.y)),
                           pack_f16(bf16lo(v.z), bf16hi(v.z)), pack_f16(bf16lo(v.w), bf16hi(v.w)));
          const int hf = c16 >> 3, cc = c16 & 7;
          *reinterpret_cast<uint4*>(qdst + hf * Cfg::kQHalfBytes + r * 128 + ((cc ^ (r & 7)) << 4)) = v;
        }
        tc::fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_full);
      }
      const uint32_t trow = tmem + t * Cfg::kTileCols + (static_cast<uint32_t>((warp & 3) * 32) << 16);
      const float sl2 = a.scale_log2;
      float m_ref = -INFINITY, l = 0.f;  // m_ref in scaled (log2) units
      bool ok = true;
      for (int j = 0; j < mych; ++j) {
        const int sb = j & 1;
        if (!warp_wait(&s_full[t][sb], (j >> 1) & 1, &ps.abort_flag)) {
          ok = false;
          break;
        }
        tc::fence_after();
        uint32_t sr[C];
        tc::ld32(trow + D + sb * C, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tc::ld32(trow + D + sb * C + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tc::wait_ld();
        const int32_t k0 = j * C;
        float x[C];
        // the row maximum over 4 independent partial maxima (three-input max:
        // short dependence chains, one instruction per two scores)
        float pm[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) pm[u] = -INFINITY;
        // warp-uniform choice: tcgen05.ld/st below need the whole warp converged
        if (__all_sync(0xffffffffu, k0 + C - 1 <= pos)) {
#pragma unroll
          for (int c = 0; c < C; ++c) x[c] = __uint_as_float(sr[c]);
        } else {
#pragma unroll
          for (int c = 0; c < C; ++c) x[c] = k0 + c <= pos ? __uint_as_float(sr[c]) : -INFINITY;
        }
#pragma unroll
        for (int c = 0; c < C / 2; ++c) pm[c & 3] = fmax3(pm[c & 3], x[2 * c], x[2 * c + 1]);
        float mx = fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3]));
        mx *= sl2;  // scale > 0 keeps the order
        float alpha = 1.f;
        bool resc = false;
        if (mx > m_ref + 8.f) {
          alpha = fast_exp2(m_ref - mx);  // 0 while m_ref is -inf
          l *= alpha;
          m_ref = mx;
          resc = j > 0;
        }
        uint32_t ph[C / 2];
        // weights as packed pairs: (x0, x1) * scale - m in one instruction, the
        // sums in two packed partial sums (short dependence chains)
        const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(-m_ref, -m_ref);
        float2 part[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < C / 2; ++c) {
          const float2 y = ffma2(make_float2(x[2 * c], x[2 * c + 1]), sc2, nm2);
          const float2 pp = make_float2(fast_exp2(y.x), fast_exp2(y.y));
          part[c & 1] = fadd2(part[c & 1], pp);
          ph[c] = pack_f16(pp.x, pp.y);  // weights <= 2^8
        }
        l += (part[0].x + part[0].y) + (part[1].x + part[1].y);
        __syncwarp();
        tc::st32(trow + D + sb * C, ph);
        if (__any_sync(0xffffffffu, resc)) {
          // O must hold P(j-1) V(j-1) before it is rescaled (P(j-2) V(j-2) is
          // complete: it was issued before S(j), which this chunk waited for)
          if (!warp_wait(&o_bar[t], (j - 1) & 1, &ps.abort_flag)) {
            tc::wait_st();
            ok = false;
            break;
          }
          tc::fence_after();
#pragma unroll
          for (int q = 0; q < D / 32; ++q) {
            uint32_t o[32];
            __syncwarp();
            tc::ld32(trow + q * 32, o);
            tc::wait_ld();
            if (resc) {
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            }
            __syncwarp();
            tc::st32(trow + q * 32, o);
          }
        }
        __syncwarp();
        tc::wait_st();
        tc::fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[t][sb]);
      }
      // O is final once the last P V has completed; its own single-phase
      // barrier (o_bar may by then be two phases past the one a parity wait
      // would name, if this warp is slow to get here after its last arrival)
      if (ok) ok = warp_wait(&o_last[t], 0, &ps.abort_flag);
      if (ok) {
        tc::fence_after();
        const float inv = (F8 ? a.v_scale : 1.f) / l;
        if (t == ntiles_act - 1 && tok0 + TT <= n) {
          // The last tile, all rows valid: its last P V was the CTA's last MMA,
          // so the K/V stages are free. O goes there as D / 32 boxes of
          // [128 rows x 32 columns] fp32 in the TMA's 128-byte swizzle, and one
          // thread stores them with the TMA (rows = (token, head) of the
          // output's [tokens][heads][D] layout); the CTA waits only for the
          // copies' reads of shared memory.
          uint8_t* stg = sgen + Cfg::kQBytes;
#pragma unroll
          for (int q = 0; q < D / 32; ++q) {
            uint32_t o[32];
            __syncwarp();
            tc::ld32(trow + q * 32, o);
            tc::wait_ld();
#pragma unroll
            for (int e = 0; e < 8; ++e)
              *reinterpret_cast<float4*>(stg + q * (128 * 128) + r * 128 + ((e ^ (r & 7)) << 4)) =
                  make_float4(__uint_as_float(o[4 * e]) * inv, __uint_as_float(o[4 * e + 1]) * inv,
                              __uint_as_float(o[4 * e + 2]) * inv, __uint_as_float(o[4 * e + 3]) * inv);
          }
          tc::fence_proxy_async();  // generic-proxy writes -> the TMA's reads
          __syncwarp();
          if (lane == 0) mbar_arrive(&o_staged);
          if ((warp & 3) == 0) {
            if (warp_wait(&o_staged, 0, &ps.abort_flag) && lane == 0) {
#pragma unroll
              for (int q = 0; q < D / 32; ++q)
                tma_store_3d(&tmo, smem_u32(stg) + q * (128 * 128), q * 32, g * G, q0 + tok0);
              bulk_commit();
              bulk_wait_read();
            }
            __syncwarp();
          }
        } else {
        // O leaves through shared memory, 32 columns at a time, staged in the
        // tile's Q area (free: every MMA of the tile has completed). Each
        // thread writes its row's 128 bytes (16-byte pieces rotated by row: no
        // bank conflicts), then the warp stores its 32 rows as whole 128-byte
        // segments, eight lanes per row, four rows per instruction, instead of
        // one 16-byte piece of 32 different rows per instruction.
        uint8_t* stg = sgen + t * Cfg::kQTileBytes + (warp & 3) * 32 * 128;
        const int pc = lane & 7;  // store phase: 16-byte piece of the row
#pragma unroll
        for (int q = 0; q < D / 32; ++q) {
          uint32_t o[32];
          __syncwarp();
          tc::ld32(trow + q * 32, o);
          tc::wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e)
            *reinterpret_cast<float4*>(stg + lane * 128 + ((e ^ (lane & 7)) << 4)) =
                make_float4(__uint_as_float(o[4 * e]) * inv, __uint_as_float(o[4 * e + 1]) * inv,
                            __uint_as_float(o[4 * e + 2]) * inv, __uint_as_float(o[4 * e + 3]) * inv);
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int rw = 4 * i + (lane >> 3);         // row within the warp's 32
            const int rr = (warp & 3) * 32 + rw;        // row within the tile
            const int32_t tk = tok0 + rr / G;
            if (tk < n) {
              const int64_t orr = (static_cast<int64_t>(q0) + tk) * a.hq + g * G + rr % G;
              *reinterpret_cast<float4*>(a.out + orr * D + q * 32 + pc * 4) =
                  *reinterpret_cast<const float4*>(stg + rw * 128 + ((pc ^ (rw & 7)) << 4));
            }
          }
        }
        }
      }
      tc::fence_before();
    }
  }
  __syncthreads();
  if (warp == Cfg::kMmaWarp) {
    tc::fence_after();
    tc::dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace pa
