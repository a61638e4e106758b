// Paged decode attention on the CUDA cores.
//
// P2 = "PagedAttention：操作系统级 KV 缓存虚拟内存管理".
//   §1.1  out = softmax(scale * q K^T) V.
//   §3.2.2 step 4, §4.1  every logical block is visited through the block
//         table; one CTA owns one attention head group; the query stays in
//         registers; the softmax is accumulated tile by tile (online softmax).
//   §4.2  each block is contiguous, so it is moved with wide copies.
//
// B200 design:
//   * CTA = (kv head g, sequence s, partition p); grid (Hkv, B, partitions), so
//     partition 0 of every sequence is dispatched before any later (shorter
//     or empty) partition. All G = Hq/Hkv query heads of the group are handled
//     together, so each K/V row is read from HBM once.
//   * Warp 4 is the producer: it reads the chunk's block ids and starts one
//     TMA bulk copy (cp.async.bulk) per (block, head) tile of K and of V into a
//     ring of S stages of 64 tokens, with an L2 evict-first hint (each K/V byte
//     is read once per step). Warps 0-3 consume: "full" mbarriers carry the
//     TMA byte counts, "empty" mbarriers collect one arrival per consumer
//     warp, so no warp ever waits on a CTA-wide barrier inside the loop.
//   * Consumer warp w owns tokens [16w, 16w+16) of a chunk. Each lane reads 16
//     bytes (8 bf16 or 4 fp32; 8 bytes = 8 e4m3 codes for fp8) of a row per load, so LPR = D / (elements per
//     load) lanes cover a row and one warp load covers RPW = 32/LPR rows. Per-lane partial
//     dot products of the NV = 16/RPW tokens a lane touched are summed across
//     the LPR lanes of its row group with a transposing butterfly (each step
//     halves the values a lane carries), after which lane (h, sub) holds the
//     score of token ((sub >> (log LPR - log NV)) * RPW + h).
//   * Online softmax in base 2 per warp, fp32 throughout; at the end the row
//     groups and then the warps are merged, and the CTA writes either the
//     normalised row (one partition) or its (m, l, o) partials.
//   * Tokens at or past the context length are never multiplied: their scores
//     are replaced by -inf and their V rows are skipped, so padding (even NaN)
//     in a partly filled last block cannot leak into the result.
#pragma once

#include "decode_common.cuh"

namespace pa {

__host__ __device__ constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x >> 1); }

// Bytes of a row one lane loads: 16, except 8 for fp8 so that a lane holds
// the same 8 elements (and registers) as with bf16.
template <typename T>
struct LaneBytes {
  static constexpr int value = Elem<T>::bytes == 1 ? 8 : 16;
};

// One lane's bytes of a row -> floats.
template <typename T>
__device__ __forceinline__ void load16(const T* p, float (&f)[LaneBytes<T>::value / Elem<T>::bytes]);

template <>
__device__ __forceinline__ void load16<float>(const float* p, float (&f)[4]) {
  const float4 x = *reinterpret_cast<const float4*>(p);
  f[0] = x.x;
  f[1] = x.y;
  f[2] = x.z;
  f[3] = x.w;
}
template <>
__device__ __forceinline__ void load16<__nv_bfloat16>(const __nv_bfloat16* p, float (&f)[8]) {
  const uint4 x = *reinterpret_cast<const uint4*>(p);
  f[0] = bf16lo(x.x);
  f[1] = bf16hi(x.x);
  f[2] = bf16lo(x.y);
  f[3] = bf16hi(x.y);
  f[4] = bf16lo(x.z);
  f[5] = bf16hi(x.z);
  f[6] = bf16lo(x.w);
  f[7] = bf16hi(x.w);
}
template <>
__device__ __forceinline__ void load16<__nv_fp8_e4m3>(const __nv_fp8_e4m3* p, float (&f)[8]) {
  const uint2 x = *reinterpret_cast<const uint2*>(p);
  const uint32_t w[2] = {x.x, x.y};
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const float2 a = fp8x2_to_float2(static_cast<uint16_t>(w[u] & 0xffffu));
    const float2 b = fp8x2_to_float2(static_cast<uint16_t>(w[u] >> 16));
    f[4 * u + 0] = a.x;
    f[4 * u + 1] = a.y;
    f[4 * u + 2] = b.x;
    f[4 * u + 3] = b.y;
  }
}

template <>
__device__ __forceinline__ void load16<int8_t>(const int8_t* p, float (&f)[8]) {
  const uint2 x = *reinterpret_cast<const uint2*>(p);
  float a[4], b[4];
  s8x4_to_float(x.x, a);
  s8x4_to_float(x.y, b);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[e] = a[e];
    f[4 + e] = b[e];
  }
}

// Sum NV values over the LPR lanes of a row group; lanes halve the values they
// carry at each of the first log2(NV) steps. Returns the full sum of value
// j = (sub >> (log LPR - log NV)) & (NV - 1).
template <int NV, int LPR>
__device__ __forceinline__ float transposed_sum(const float (&in)[NV], int sub) {
  float v[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) v[i] = in[i];
#pragma unroll
  for (int step = 0; step < ilog2(LPR); ++step) {
    const int o = LPR >> (step + 1);
    const int cnt = NV >> step;
    if (cnt > 1) {
      const bool up = sub & o;
#pragma unroll
      for (int u = 0; u < cnt / 2; ++u) {
        const float send = up ? v[u] : v[u + cnt / 2];
        const float keep = up ? v[u + cnt / 2] : v[u];
        v[u] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
  return v[0];
}

template <typename T, int D>
struct SimtCfg {
  static constexpr int kConsumerWarps = 4;
  static constexpr int kThreads = 32 * (kConsumerWarps + 1);
  static constexpr int kTokPerWarp = 16;
  static constexpr int kChunk = kTokPerWarp * kConsumerWarps;  // tokens per stage
  static constexpr int kEPL = LaneBytes<T>::value / Elem<T>::bytes;  // elements per lane load
  static constexpr int kLPR = D / kEPL;                        // lanes per row
  static constexpr int kRPW = 32 / kLPR;                       // rows per warp load
  static constexpr int kNV = kTokPerWarp / kRPW;               // token partials per lane
  static constexpr int kStageBytes = 2 * kChunk * D * Elem<T>::bytes;
  static constexpr int kStages = kStageBytes <= 16384 ? 4 : 2;  // 2 x 32 KB at D 128 bf16: 3 CTAs per SM
  static constexpr int kSmemBytes = kStages * kStageBytes;
  static_assert(kNV <= kLPR, "butterfly needs at least as many lanes as values");
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(SimtCfg<T, D>::kThreads) decode_simt_kernel(const DecodeArgs a) {
  using Cfg = SimtCfg<T, D>;
  constexpr int NW = Cfg::kConsumerWarps, C = Cfg::kChunk, S = Cfg::kStages, EPL = Cfg::kEPL, LPR = Cfg::kLPR,
                RPW = Cfg::kRPW, NV = Cfg::kNV, TPW = Cfg::kTokPerWarp;
  constexpr int REP = ilog2(LPR) - ilog2(NV);  // low lane bits that replicate a token after the butterfly
  static_assert(NW * G * (D + 2) * 4 <= Cfg::kSmemBytes, "merge buffer must fit in the stage ring");

  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ PipeSmem<S> ps;
  T* sK = reinterpret_cast<T*>(smem);
  T* sV = sK + S * C * D;

  const int g = blockIdx.x, p = blockIdx.z;
  const int s = grid_seq(a, blockIdx.y, g == 0 && p == 0 && threadIdx.x == 0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  Part pt;
  if (!cta_part<G, D>(a, g, s, p, tid, Cfg::kThreads, pt)) return;
  const int nchunks = (pt.ntok + C - 1) / C;
  const int hq0 = g * G;

  if (tid == 0) pipe_init<S>(ps, NW);
  __syncthreads();

  float m[G], lsum[G], acc[G][EPL];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    lsum[h] = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[h][e] = 0.f;
  }
  const int hrow = lane / LPR, sub = lane % LPR;

  if (warp == NW) {
    // ---- producer ----
    // fused KV append: the new row is loaded now and stored before the last
    // chunk's copies, which read it
    const bool do_append = a.slot_mapping && pt.last;
    AppendRow<T, D> ar;
    if (do_append) ar.load(a, s, g, lane);
    const int64_t table_row = static_cast<int64_t>(s) * a.max_blocks;
    const uint32_t tile_bytes = static_cast<uint32_t>(a.bs) * D * Elem<T>::bytes;
    const T* kc = static_cast<const T*>(a.kc);
    const T* vc = static_cast<const T*>(a.vc);
    const uint64_t pol = kv_stream_policy();
    pipe_produce<S>(ps, nchunks, [&](int i, int st) {
      if (do_append) ar.before_chunk(a, i, nchunks, lane);
      const int32_t c0 = pt.t0 + i * C;
      const int32_t nb = (min(C, pt.t1 - c0) + a.bs - 1) / a.bs;  // <= 64 (C = 64, bs >= 1)
      int32_t blk[2] = {-1, -1};
      bool ok[2] = {false, false};
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int j = lane + 32 * u;
        if (j < nb) {
          blk[u] = __ldg(a.tables + table_row + c0 / a.bs + j);
          ok[u] = blk[u] >= 0 && blk[u] < a.num_blocks;
          if (!ok[u]) record_error(PA_ERR_DEVICE_BOUNDS, blk[u]);
        }
      }
      const int cnt = __popc(__ballot_sync(0xffffffffu, ok[0])) + __popc(__ballot_sync(0xffffffffu, ok[1]));
      if (lane == 0) mbar_arrive_expect_tx(&ps.full[st], 2u * cnt * tile_bytes);
      __syncwarp();
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (ok[u]) {
          const int64_t off = (static_cast<int64_t>(blk[u]) * a.hkv + g) * a.bs * D;
          const int32_t row = (lane + 32 * u) * a.bs;
          bulk_g2s(sK + (st * C + row) * D, kc + off, tile_bytes, &ps.full[st], pol);
          bulk_g2s(sV + (st * C + row) * D, vc + off, tile_bytes, &ps.full[st], pol);
        }
      }
      if (do_append) ar.after_chunk(a, i, nchunks, lane);
    });
  } else {
    // ---- consumers ----
    float qv[G][EPL];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      using QT = typename QueryOf<T>::type;
      const QT* qp = static_cast<const QT*>(a.q) + (static_cast<int64_t>(s) * a.hq + hq0 + h) * D + sub * EPL;
#pragma unroll
      for (int e = 0; e < EPL; ++e) qv[h][e] = to_f<QT>(qp[e]) * a.scale_log2;
    }
    const int my_j = (sub >> REP) & (NV - 1);
    const int my_tok = my_j * RPW + hrow;        // token (within the warp's 16) whose score this lane holds
    const bool counts = (sub & ((1 << REP) - 1)) == 0;

    for (int i = 0; i < nchunks; ++i) {
      const int st = i % S;
      if (!pipe_wait(&ps.full[st], (i / S) & 1, &ps.abort_flag)) break;
      const int nv = min(TPW, min(C, pt.ntok - i * C) - warp * TPW);  // warp-uniform
      if (nv > 0) {
        const T* Kw = sK + (st * C + warp * TPW) * D + sub * EPL;
        const T* Vw = sV + (st * C + warp * TPW) * D + sub * EPL;
        float part[G][NV];
#pragma unroll
        for (int j = 0; j < NV; ++j) {
          const int tok = j * RPW + hrow;
          float kf[EPL];
          if (tok < nv) {
            load16<T>(Kw + tok * D, kf);
          } else {
#pragma unroll
            for (int e = 0; e < EPL; ++e) kf[e] = 0.f;
          }
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float d0 = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) d0 = fmaf(qv[h][e], kf[e], d0);
            part[h][j] = d0;
          }
        }
        float pj[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float sc = transposed_sum<NV, LPR>(part[h], sub);
          sc = my_tok < nv ? sc : -INFINITY;
          const float cm = warp_max(sc);
          const float mn = fmaxf(m[h], cm);
          const float alpha = exp2f(m[h] - mn);
          pj[h] = exp2f(sc - mn);
          lsum[h] = lsum[h] * alpha + (counts ? pj[h] : 0.f);
#pragma unroll
          for (int e = 0; e < EPL; ++e) acc[h][e] *= alpha;
          m[h] = mn;
        }
#pragma unroll
        for (int j = 0; j < NV; ++j) {
          const int tok = j * RPW + hrow;
          const int src = hrow * LPR + (j << REP);
          float w[G];
#pragma unroll
          for (int h = 0; h < G; ++h) w[h] = __shfl_sync(0xffffffffu, pj[h], src);
          if (tok < nv) {
            float vf[EPL];
            load16<T>(Vw + tok * D, vf);
#pragma unroll
            for (int h = 0; h < G; ++h)
#pragma unroll
              for (int e = 0; e < EPL; ++e) acc[h][e] = fmaf(w[h], vf[e], acc[h][e]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ps.empty[st]);
    }
    // fold the row groups of the warp together (and apply an fp8 V scale)
#pragma unroll
    for (int h = 0; h < G; ++h) {
      lsum[h] = warp_sum(lsum[h]);
#pragma unroll
      for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[h][e] += __shfl_xor_sync(0xffffffffu, acc[h][e], o);
      if (Elem<T>::bytes == 1) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[h][e] *= a.v_scale;
      }
    }
  }

  __syncthreads();  // every copy consumed; the stage ring is free
  if (ps.abort_flag) return;

  float* wm = reinterpret_cast<float*>(smem);
  float* wl = wm + NW * G;
  float* wacc = wl + NW * G;
  if (warp < NW) {
    if (lane == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        wm[warp * G + h] = m[h];
        wl[warp * G + h] = lsum[h];
      }
    }
    if (hrow == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < EPL; ++e) wacc[(warp * G + h) * D + sub * EPL + e] = acc[h][e];
    }
  }
  __syncthreads();
  merge_warps_and_store<G, D, NW>(a, wm, wl, wacc, s, p, hq0, pt.nparts, pt.npre, tid, Cfg::kThreads);
}

}  // namespace pa
