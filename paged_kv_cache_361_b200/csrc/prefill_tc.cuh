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
// a kv head read every K/V tile once. Six warps:
//   warp 4     TMA producer: swizzled [bs x 64] boxes of K and V, 64 keys per
//              stage (the ring and its full/empty barriers of the decode path).
//   warp 5     allocates TMEM; one lane issues every MMA:
//                S_j = Q K_j^T        (M 128, N 64, K = D; A and B in shared
//                                      memory, K-major) into TMEM buffer j % 2
//                O  += P_j V_j        (M 128, N = D, K 64; A = P from TMEM,
//                                      B = V in shared memory, N-major)
//              S_{j+1} is issued before O += P_j V_j so the tensor core works
//              while the softmax warps handle chunk j. Completions reach the
//              other warps through tcgen05.commit on mbarriers.
//   warps 0-3  one thread per row (TMEM lane): load the row's Q into shared
//              memory; per chunk read S from TMEM, mask causally, keep the
//              running maximum m and sum l in base 2, write P back into the
//              S buffer as a bf16 high part and a bf16 remainder (two MMAs
//              for P V keep ~16 mantissa bits of each weight); at the end read
//              O, divide by l, store fp32.
// The running maximum is moved (and O rescaled in TMEM) only when a row's
// maximum grows by more than 8 in log2 units, so weights stay below 2^8 and
// most chunks never touch O; the result is the same softmax.
#pragma once

#include "prefill_mma.cuh"
#include "tcgen05.cuh"

namespace pa {

template <int D>
struct TcCfg {
  static constexpr int kRows = 128;                        // query rows per tile (MMA M)
  static constexpr int kChunk = 64;                        // keys per stage
  static constexpr int kHalves = D / 64;                   // 128-byte column boxes per row
  static constexpr int kHalfBytes = kChunk * 128;          // one box column of K or V in a stage
  static constexpr int kTileBytes = kHalves * kHalfBytes;  // K (or V) of one stage
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStages = 4;
  static constexpr int kQHalfBytes = kRows * 128;
  static constexpr int kQBytes = kHalves * kQHalfBytes;
  static constexpr int kSmemBytes = 1024 + kQBytes + kStages * kStageBytes;
  static constexpr int kThreads = 192;
  static constexpr uint32_t kTmemCols = 256;  // O: D columns; S/P: two buffers of 64 after it
  static constexpr uint32_t kColO = 0;
  static constexpr uint32_t kColS = D;
  static_assert(kColS + 2 * kChunk <= kTmemCols, "TMEM columns");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

// All lanes wait; the warp proceeds only if every lane saw the phase.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const bool ok = pipe_wait(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

template <int D, int G>
__global__ void __launch_bounds__(192, 1) prefill_tc_kernel(const __grid_constant__ CUtensorMap tmk,
                                                            const __grid_constant__ CUtensorMap tmv,
                                                            const PrefillArgs a) {
  using Cfg = TcCfg<D>;
  constexpr int S = Cfg::kStages, C = Cfg::kChunk, TT = Cfg::kRows / G;

  extern __shared__ uint8_t smem_raw[];
  __shared__ PipeSmem<S> ps;
  __shared__ uint64_t q_full, s_full[2], p_full[2], o_bar, drain;
  __shared__ uint32_t tmem_base_sh;
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);  // generic pointer to sbase
  const uint32_t qs = sbase;                 // Q: kHalves x [128 rows x 128 B], swizzled
  const uint32_t kv0 = sbase + Cfg::kQBytes;  // stage st: K halves, then V halves

  const int g = blockIdx.x, s = blockIdx.z;
  const int tile = a.ntiles - 1 - static_cast<int>(blockIdx.y);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int32_t q0 = __ldg(a.cu_q + s);
  int32_t n = __ldg(a.cu_q + s + 1) - q0;
  int32_t L = __ldg(a.lens + s);
  if (L < 0 || L > a.max_ctx || n < 0 || n > L) {
    if (tid == 0 && g == 0 && tile == 0) record_error(PA_ERR_DEVICE_BOUNDS, L);
    L = L < 0 ? 0 : (L > a.max_ctx ? a.max_ctx : L);
    n = n < 0 ? 0 : (n > L ? L : n);
  }
  const int32_t tok0 = tile * TT;
  if (tok0 >= n) return;
  const int32_t tok_end = min(tok0 + TT, n);
  const int32_t base = L - n;           // position of new token 0
  const int32_t kend = base + tok_end;  // keys 0 .. kend-1 are needed (kend >= 1)
  const int nchunks = (kend + C - 1) / C;
  const int64_t table_row = static_cast<int64_t>(s) * a.max_blocks;

  if (tid == 0) {
    mbar_init(&q_full, 4);
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(&p_full[0], 4);
    mbar_init(&p_full[1], 4);
    mbar_init(&o_bar, 1);
    mbar_init(&drain, 1);
    pipe_init<S>(ps, 1);  // empty stages are released by one tcgen05.commit
  }
  if (warp == 5) {
    tc::alloc(smem_u32(&tmem_base_sh), Cfg::kTmemCols);
    tc::relinquish();
    tc::fence_before();
  }
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 4) {
    // ---- producer ----
    const uint32_t box_bytes = static_cast<uint32_t>(a.bs) * 128u;
    const uint64_t pol = l2_evict_last_policy();  // later tiles of this sequence read the same keys
    pipe_produce<S>(ps, nchunks, [&](int i, int st) {
      const int32_t c0 = i * C;
      const int32_t nb = (min(C, kend - c0) + a.bs - 1) / a.bs;  // <= 8 (bs >= 8)
      int32_t blk = -1;
      bool ok = false;
      if (lane < nb) {
        blk = __ldg(a.tables + table_row + c0 / a.bs + lane);
        ok = blk >= 0 && blk < a.num_blocks;
        if (!ok) record_error(PA_ERR_DEVICE_BOUNDS, blk);
      }
      const unsigned okmask = __ballot_sync(0xffffffffu, ok);
      if (lane == 0) mbar_arrive_expect_tx(&ps.full[st], 2u * Cfg::kHalves * __popc(okmask) * box_bytes);
      __syncwarp();
      if (ok) {
        const int32_t y = (blk * a.hkv + g) * a.bs;
        const uint32_t kdst = kv0 + st * Cfg::kStageBytes + lane * box_bytes;
#pragma unroll
        for (int hf = 0; hf < Cfg::kHalves; ++hf) {
          tma_load_2d(kdst + hf * Cfg::kHalfBytes, &tmk, hf * 64, y, &ps.full[st], pol);
          tma_load_2d(kdst + Cfg::kTileBytes + hf * Cfg::kHalfBytes, &tmv, hf * 64, y, &ps.full[st], pol);
        }
      }
    });
  } else if (warp == 5) {
    // ---- MMA issuer ----
    if (lane == 0) {
      constexpr uint32_t kIdS = tc::idesc_bf16(Cfg::kRows, C, false);
      constexpr uint32_t kIdPV = tc::idesc_bf16(Cfg::kRows, D, true);
      auto issue_pv = [&](int i) -> bool {
        const int sb = i & 1, st = i % S;
        if (!pipe_wait(&p_full[sb], (i >> 1) & 1, &ps.abort_flag)) return false;
        tc::fence_after();
        const uint32_t vbase = kv0 + st * Cfg::kStageBytes + Cfg::kTileBytes;
        const uint32_t tp = tmem + Cfg::kColS + sb * C;  // P high part: 32 columns, remainder: the next 32
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks) {
          // V is N-major: 8-key groups 1024 B apart, the two 64-column halves
          // kHalfBytes apart (one half when D = 64: the offset is then unused)
          const uint64_t bd = tc::smem_desc(vbase + ks * 16 * 128, Cfg::kHalves > 1 ? Cfg::kHalfBytes : 1024, 1024);
          tc::mma_ts(tmem + Cfg::kColO, tp + ks * 8, bd, kIdPV, i > 0 || ks > 0);
          tc::mma_ts(tmem + Cfg::kColO, tp + C / 2 + ks * 8, bd, kIdPV, true);
        }
        tc::commit(smem_u32(&ps.empty[st]));
        tc::commit(smem_u32(&o_bar));
        return true;
      };
      bool ok = pipe_wait(&q_full, 0, &ps.abort_flag);
      tc::fence_after();
      for (int j = 0; ok && j < nchunks; ++j) {
        const int st = j % S, sb = j & 1;
        if (!pipe_wait(&ps.full[st], (j / S) & 1, &ps.abort_flag)) {
          ok = false;
          break;
        }
        tc::fence_after();
        const uint32_t kbase = kv0 + st * Cfg::kStageBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32u;  // 16 dims = 32 B along the swizzled 128-byte row
          const uint64_t qd = tc::smem_desc(qs + (kk >> 2) * Cfg::kQHalfBytes + off, 16, 1024);
          const uint64_t kd = tc::smem_desc(kbase + (kk >> 2) * Cfg::kHalfBytes + off, 16, 1024);
          tc::mma_ss(tmem + Cfg::kColS + sb * C, qd, kd, kIdS, kk > 0);
        }
        tc::commit(smem_u32(&s_full[sb]));
        if (j > 0) ok = issue_pv(j - 1);
      }
      if (ok) issue_pv(nchunks - 1);
      // every MMA this thread issued has finished before TMEM is released
      tc::commit(smem_u32(&drain));
      mbar_wait(&drain, 0);
    }
    __syncwarp();
  } else {
    // ---- softmax warps: thread = row = TMEM lane ----
    const int r = tid;
    const int tok = tok0 + r / G;
    const bool valid = tok < n;
    const int32_t pos = base + (valid ? tok : tok_end - 1);  // last key the row sees
    const int h = r % G;
    const int64_t orow = (static_cast<int64_t>(q0) + (valid ? tok : 0)) * a.hq + g * G + h;
    {
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) + orow * D);
#pragma unroll
      for (int c16 = 0; c16 < D / 8; ++c16) {
        const uint4 v = valid ? __ldg(src + c16) : make_uint4(0u, 0u, 0u, 0u);
        const int hf = c16 >> 3, cc = c16 & 7;
        *reinterpret_cast<uint4*>(sgen + hf * Cfg::kQHalfBytes + r * 128 + ((cc ^ (r & 7)) << 4)) = v;
      }
      tc::fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(&q_full);
    }
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nchunks; ++j) {
      const int sb = j & 1;
      if (!warp_wait(&s_full[sb], (j >> 1) & 1, &ps.abort_flag)) {
        ok = false;
        break;
      }
      tc::fence_after();
      uint32_t sr[C];
      tc::ld32(trow + Cfg::kColS + sb * C, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tc::ld32(trow + Cfg::kColS + sb * C + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tc::wait_ld();
      const int32_t k0 = j * C;
      float x[C];
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < C; ++c) {
        x[c] = k0 + c <= pos ? __uint_as_float(sr[c]) * a.scale_log2 : -INFINITY;
        mx = fmaxf(mx, x[c]);
      }
      float alpha = 1.f;
      bool resc = false;
      if (mx > m_ref + 8.f) {
        alpha = exp2f(m_ref - mx);  // 0 while m_ref is -inf
        l *= alpha;
        m_ref = mx;
        resc = j > 0;
      }
      uint32_t ph[C / 2], pl[C / 2];
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < C / 2; ++c) {
        const float p0 = exp2f(x[2 * c] - m_ref), p1 = exp2f(x[2 * c + 1] - m_ref);
        sum += p0 + p1;
        split_pair(p0, p1, ph[c], pl[c]);
      }
      l += sum;
      tc::st32(trow + Cfg::kColS + sb * C, ph);
      tc::st32(trow + Cfg::kColS + sb * C + C / 2, pl);
      if (__any_sync(0xffffffffu, resc)) {
        // O must hold P_{j-1} V_{j-1} before it is rescaled
        if (!warp_wait(&o_bar, (j - 1) & 1, &ps.abort_flag)) {
          tc::wait_st();
          ok = false;
          break;
        }
        tc::fence_after();
#pragma unroll
        for (int q = 0; q < D / 32; ++q) {
          uint32_t o[32];
          tc::ld32(trow + Cfg::kColO + q * 32, o);
          tc::wait_ld();
          if (resc) {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          }
          tc::st32(trow + Cfg::kColO + q * 32, o);
        }
      }
      if (j == nchunks - 1 && kend - k0 < C) {
        // V rows past the last key may hold anything (unloaded or padding);
        // 0 * NaN would reach O, so they are zeroed before P V reads them.
        const int nvk = kend - k0;
        const int chunks16 = (C - nvk) * Cfg::kHalves * 8;
        uint8_t* vst = sgen + Cfg::kQBytes + (j % S) * Cfg::kStageBytes + Cfg::kTileBytes;
        tc::fence_proxy_async();
        for (int i = r; i < chunks16; i += 128) {
          const int row = nvk + i / (Cfg::kHalves * 8);
          const int rem = i % (Cfg::kHalves * 8);
          *reinterpret_cast<uint4*>(vst + (rem >> 3) * Cfg::kHalfBytes + row * 128 + (rem & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        tc::fence_proxy_async();
      }
      tc::wait_st();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
    }
    if (ok) ok = warp_wait(&o_bar, (nchunks - 1) & 1, &ps.abort_flag);
    if (ok) {
      tc::fence_after();
      const float inv = 1.f / l;
      float* dst = a.out + orow * D;
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        uint32_t o[32];
        tc::ld32(trow + Cfg::kColO + q * 32, o);
        tc::wait_ld();
        if (valid) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + q * 32 + e) =
                make_float4(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv,
                            __uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
        }
      }
    }
    tc::fence_before();
  }
  __syncthreads();
  if (warp == 5) {
    tc::fence_after();
    tc::dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace pa
