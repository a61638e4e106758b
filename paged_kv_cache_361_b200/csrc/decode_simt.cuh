// Paged decode attention on the CUDA cores, and the partition merge.
//
// P2 = "PagedAttention：操作系统级 KV 缓存虚拟内存管理".
//   §1.1  out = softmax(scale * q K^T) V.
//   §3.2.2 step 4, §4.1  every logical block is visited through the block
//         table; one CTA owns one attention head group; the query stays in
//         registers; the softmax is accumulated tile by tile (online softmax).
//   §4.2  each block is contiguous, so it is moved with wide copies.
//
// B200 design:
//   * CTA = (kv head g, sequence s, partition p), 4 warps. All G = Hq/Hkv query
//     heads of the group are processed together so each K/V row is read once.
//     The grid is (Hkv, B, partitions), so partition 0 of every sequence is
//     dispatched before any later (shorter or empty) partition.
//   * K/V move HBM -> shared memory as whole (block, head) tiles by the TMA
//     unit (cp.async.bulk, one instruction per tile, up to 32 in parallel from
//     one warp), into an S-stage ring of 32-token chunks guarded by mbarriers,
//     with an L2 evict-first hint (every K/V byte is read once per step).
//   * Warp w owns tokens [8w, 8w+8) of each chunk. Lane l holds dims
//     [l*VEC, l*VEC+VEC) of the query (pre-scaled by scale*log2 e) and of its
//     output accumulator. Dot products are reduced across the warp with a
//     transposing butterfly: 8 token sums in 9 shuffles, after which lane l
//     holds the score of token (l >> 2) & 7.
//   * Online softmax in base 2 per warp; warps merge through shared memory at
//     the end. With one partition the CTA writes the normalised row; otherwise
//     it writes (m, l, unnormalised o) to the workspace for decode_reduce.
//   * Tokens at or past the context length are never multiplied: their scores
//     are replaced by -inf and their V rows are skipped, so padding (even NaN)
//     in a partly filled last block cannot leak into the result.
#pragma once

#include "common.cuh"

namespace pa {

struct DecodeArgs {
  const void* q;
  const void* kc;
  const void* vc;
  const int32_t* tables;
  const int32_t* lens;
  float* out;
  float* ws_ml;   // [num_seqs][hq][max_parts][2]  (m in log2 units, l)
  float* ws_o;    // [num_seqs][hq][max_parts][D]
  int64_t num_blocks;
  int32_t num_seqs, hq, hkv, bs, max_blocks, max_ctx;
  int32_t part_tokens;  // > 0: partition size; 0: one partition per sequence
  int32_t max_parts;    // grid.z
  float scale_log2;     // scale * log2(e)
};

template <typename T>
struct Elem;
template <>
struct Elem<float> {
  static constexpr int bytes = 4;
};
template <>
struct Elem<__nv_bfloat16> {
  static constexpr int bytes = 2;
};

// VEC consecutive elements of a row -> floats.
template <typename T, int VEC>
__device__ __forceinline__ void load_row(const T* p, float (&f)[VEC]);

template <>
__device__ __forceinline__ void load_row<float, 4>(const float* p, float (&f)[4]) {
  float4 x = *reinterpret_cast<const float4*>(p);
  f[0] = x.x; f[1] = x.y; f[2] = x.z; f[3] = x.w;
}
template <>
__device__ __forceinline__ void load_row<float, 2>(const float* p, float (&f)[2]) {
  float2 x = *reinterpret_cast<const float2*>(p);
  f[0] = x.x; f[1] = x.y;
}
template <>
__device__ __forceinline__ void load_row<__nv_bfloat16, 4>(const __nv_bfloat16* p, float (&f)[4]) {
  uint2 x = *reinterpret_cast<const uint2*>(p);
  f[0] = bf16lo(x.x); f[1] = bf16hi(x.x); f[2] = bf16lo(x.y); f[3] = bf16hi(x.y);
}
template <>
__device__ __forceinline__ void load_row<__nv_bfloat16, 2>(const __nv_bfloat16* p, float (&f)[2]) {
  uint32_t x = *reinterpret_cast<const uint32_t*>(p);
  f[0] = bf16lo(x); f[1] = bf16hi(x);
}

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// Context length of sequence s, clamped to [0, max_ctx]; an out-of-range value
// is recorded once (by the CTA that owns head 0 / partition 0).
__device__ __forceinline__ int32_t load_len(const DecodeArgs& a, int32_t s, bool report) {
  int32_t L = __ldg(a.lens + s);
  if (L < 0 || L > a.max_ctx) {
    if (report) record_error(PA_ERR_DEVICE_BOUNDS, L);
    L = L < 0 ? 0 : a.max_ctx;
  }
  return L;
}

template <typename T, int D>
struct SimtCfg {
  static constexpr int kWarps = 4;
  static constexpr int kThreads = 128;
  static constexpr int kChunk = 32;                    // tokens per pipeline stage
  static constexpr int kTokPerWarp = kChunk / kWarps;  // 8
  static constexpr int kVec = D / 32;
  static constexpr int kStageBytes = 2 * kChunk * D * Elem<T>::bytes;  // K + V
  static constexpr int kStages = kStageBytes <= 16384 ? 4 : 3;
  static constexpr int kSmemBytes = kStages * kStageBytes;
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(128) decode_simt_kernel(const DecodeArgs a) {
  using Cfg = SimtCfg<T, D>;
  constexpr int NW = Cfg::kWarps, C = Cfg::kChunk, TPW = Cfg::kTokPerWarp, VEC = Cfg::kVec, S = Cfg::kStages;
  static_assert(TPW == 8, "the butterfly below reduces 8 token sums");
  static_assert(NW * G * (D + 2) * 4 <= Cfg::kSmemBytes, "merge buffer must fit in the stage ring");

  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t bars[S];
  T* sK = reinterpret_cast<T*>(smem);
  T* sV = sK + S * C * D;

  const int g = blockIdx.x, s = blockIdx.y, p = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int32_t L = load_len(a, s, g == 0 && p == 0 && tid == 0);
  const int32_t P = a.part_tokens > 0 ? a.part_tokens : (L > 0 ? L : 1);
  const int32_t t0 = p * P;
  const int32_t hq0 = g * G;

  if (L == 0) {
    if (p == 0)
      for (int idx = tid; idx < G * D; idx += Cfg::kThreads)
        a.out[(static_cast<int64_t>(s) * a.hq + hq0) * D + idx] = 0.f;
    return;
  }
  if (t0 >= L) return;
  const int32_t t1 = min(t0 + P, L);
  const int32_t ntok = t1 - t0;
  const int32_t nchunks = (ntok + C - 1) / C;
  const int32_t nparts = a.part_tokens > 0 ? (L + P - 1) / P : 1;

  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < S; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  __syncthreads();

  const int64_t table_row = static_cast<int64_t>(s) * a.max_blocks;
  const uint32_t tile_bytes = static_cast<uint32_t>(a.bs) * D * Elem<T>::bytes;
  const T* kc = static_cast<const T*>(a.kc);
  const T* vc = static_cast<const T*>(a.vc);
  const uint64_t pol = l2_evict_first_policy();

  // Warp 0: load the block ids of chunk i (one per lane) and start their copies.
  auto issue = [&](int i) {
    const int32_t c0 = t0 + i * C;
    const int32_t n = min(C, t1 - c0);
    const int32_t nb = (n + a.bs - 1) / a.bs;
    const int st = i % S;
    int32_t blk = -1;
    bool ok = false;
    if (lane < nb) {
      blk = __ldg(a.tables + table_row + c0 / a.bs + lane);
      ok = blk >= 0 && blk < a.num_blocks;
      if (!ok) record_error(PA_ERR_DEVICE_BOUNDS, blk);
    }
    const unsigned okmask = __ballot_sync(0xffffffffu, ok);
    if (lane == 0) mbar_arrive_expect_tx(&bars[st], 2u * __popc(okmask) * tile_bytes);
    __syncwarp();
    if (ok) {
      const int64_t off = (static_cast<int64_t>(blk) * a.hkv + g) * a.bs * D;
      const int32_t row = lane * a.bs;
      bulk_g2s(sK + (st * C + row) * D, kc + off, tile_bytes, &bars[st], pol);
      bulk_g2s(sV + (st * C + row) * D, vc + off, tile_bytes, &bars[st], pol);
    }
  };

  if (warp == 0) {
    const int npro = nchunks < S ? nchunks : S;
    for (int i = 0; i < npro; ++i) issue(i);
  }

  // Query rows of this group, pre-scaled so that exp2 gives e^(scale * q.k).
  float qv[G][VEC];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const T* qp = static_cast<const T*>(a.q) + (static_cast<int64_t>(s) * a.hq + hq0 + h) * D + lane * VEC;
#pragma unroll
    for (int e = 0; e < VEC; ++e) qv[h][e] = to_f<T>(qp[e]) * a.scale_log2;
  }

  float m[G], lsum[G], acc[G][VEC];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    lsum[h] = 0.f;
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[h][e] = 0.f;
  }

  const int jj = (lane >> 2) & 7;  // token of this lane after the butterfly
  bool failed = false;
  int i = 0;
  for (; i < nchunks; ++i) {
    const int st = i % S;
    const bool ok = mbar_wait(&bars[st], (i / S) & 1);
    if (ok) {
      const int nvalid = min(C, ntok - i * C) - warp * TPW;  // warp-uniform
      if (nvalid > 0) {
        const T* Kw = sK + (st * C + warp * TPW) * D + lane * VEC;
        const T* Vw = sV + (st * C + warp * TPW) * D + lane * VEC;
        float part[G][TPW];
#pragma unroll
        for (int j = 0; j < TPW; ++j) {
          float kf[VEC];
          if (j < nvalid) {
            load_row<T, VEC>(Kw + j * D, kf);
          } else {
#pragma unroll
            for (int e = 0; e < VEC; ++e) kf[e] = 0.f;
          }
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float d0 = 0.f;
#pragma unroll
            for (int e = 0; e < VEC; ++e) d0 = fmaf(qv[h][e], kf[e], d0);
            part[h][j] = d0;
          }
        }
        float pj[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          // transposing butterfly: 8 sums over 32 lanes -> lane holds token jj
          const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
          float r4[4], r2[2];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float send = b4 ? part[h][u] : part[h][u + 4];
            const float keep = b4 ? part[h][u + 4] : part[h][u];
            r4[u] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
          }
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const float send = b3 ? r4[u] : r4[u + 2];
            const float keep = b3 ? r4[u + 2] : r4[u];
            r2[u] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
          }
          float sc;
          {
            const float send = b2 ? r2[0] : r2[1];
            const float keep = b2 ? r2[1] : r2[0];
            sc = keep + __shfl_xor_sync(0xffffffffu, send, 4);
          }
          sc += __shfl_xor_sync(0xffffffffu, sc, 2);
          sc += __shfl_xor_sync(0xffffffffu, sc, 1);
          sc = jj < nvalid ? sc : -INFINITY;
          float cm = fmaxf(sc, __shfl_xor_sync(0xffffffffu, sc, 4));
          cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 8));
          cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 16));
          const float mn = fmaxf(m[h], cm);
          const float alpha = exp2f(m[h] - mn);
          pj[h] = exp2f(sc - mn);
          lsum[h] = lsum[h] * alpha + ((lane & 3) == 0 ? pj[h] : 0.f);
#pragma unroll
          for (int e = 0; e < VEC; ++e) acc[h][e] *= alpha;
          m[h] = mn;
        }
#pragma unroll
        for (int j = 0; j < TPW; ++j) {
          if (j < nvalid) {
            float vf[VEC];
            load_row<T, VEC>(Vw + j * D, vf);
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float w = __shfl_sync(0xffffffffu, pj[h], j << 2);
#pragma unroll
              for (int e = 0; e < VEC; ++e) acc[h][e] = fmaf(w, vf[e], acc[h][e]);
            }
          }
        }
      }
    }
    failed = __syncthreads_or(!ok);
    if (failed) break;
    if (warp == 0 && i + S < nchunks) issue(i + S);
  }

  if (failed) {
    // Let the copies already started land before the CTA exits.
    if (tid == 0)
      for (int j = i; j < nchunks && j < i + S; ++j) mbar_wait(&bars[j % S], (j / S) & 1);
    return;
  }

#pragma unroll
  for (int h = 0; h < G; ++h) lsum[h] = warp_sum(lsum[h]);

  // Merge the warps (the stage ring is free: every issued copy was consumed).
  float* wm = reinterpret_cast<float*>(smem);
  float* wl = wm + NW * G;
  float* wacc = wl + NW * G;
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      wm[warp * G + h] = m[h];
      wl[warp * G + h] = lsum[h];
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < VEC; ++e) wacc[(warp * G + h) * D + lane * VEC + e] = acc[h][e];
  __syncthreads();

  for (int idx = tid; idx < G * D; idx += Cfg::kThreads) {
    const int h = idx / D, d = idx - h * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, wm[w * G + h]);
    float l = 0.f, o = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float f = exp2f(wm[w * G + h] - M);
      l = fmaf(wl[w * G + h], f, l);
      o = fmaf(wacc[(w * G + h) * D + d], f, o);
    }
    const int64_t row = static_cast<int64_t>(s) * a.hq + hq0 + h;
    if (nparts == 1) {
      a.out[row * D + d] = o / l;
    } else {
      const int64_t prow = row * a.max_parts + p;
      a.ws_o[prow * D + d] = o;
      if (d == 0) {
        a.ws_ml[prow * 2] = M;
        a.ws_ml[prow * 2 + 1] = l;
      }
    }
  }
}

// Merge the partitions of one (sequence, query head):
//   M = max_p m_p,  out = sum_p o_p 2^(m_p - M) / sum_p l_p 2^(m_p - M).
// Grid (hq, num_seqs), D threads. Sequences with one partition were written
// by the decode kernel and are skipped.
template <int D>
__global__ void __launch_bounds__(D) decode_reduce_kernel(const DecodeArgs a) {
  const int hq = blockIdx.x, s = blockIdx.y, d = threadIdx.x;
  const int32_t L = load_len(a, s, false);
  const int32_t P = a.part_tokens;
  const int32_t nparts = (L + P - 1) / P;
  if (nparts <= 1) return;
  const int64_t row = static_cast<int64_t>(s) * a.hq + hq;
  const float* ml = a.ws_ml + row * a.max_parts * 2;
  const float* o = a.ws_o + row * a.max_parts * D;
  float M = -INFINITY;
  for (int q = 0; q < nparts; ++q) M = fmaxf(M, ml[2 * q]);
  float l = 0.f, acc = 0.f;
  for (int q = 0; q < nparts; ++q) {
    const float f = exp2f(ml[2 * q] - M);
    l = fmaf(ml[2 * q + 1], f, l);
    acc = fmaf(o[static_cast<int64_t>(q) * D + d], f, acc);
  }
  a.out[row * D + d] = acc / l;
}

}  // namespace pa
