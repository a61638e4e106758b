// KV append (slot-mapped scatter) and copy-on-write block copy.
//
// P2 = "PagedAttention：操作系统级 KV 缓存虚拟内存管理".
//   reshape_and_cache: P2 §3.2.2 step 3 (write the new token's K, V at its
//     block position) and §3.2.1 (a prompt's K, V written into its blocks).
//   copy_blocks: P2 §3.4 (a shared block is copied before it is written).
// Both are bit copies bound by HBM bandwidth. Every thread moves 16-byte
// vectors; consecutive threads touch consecutive 16-byte chunks of one row (or
// one block), so every warp access is a run of full 32-byte sectors. Rows of a
// (block, head) tile are contiguous because the cache is [block][head][offset][dim]
// (P2 §4.2: each block is a contiguous, vector-loadable region).
#pragma once

#include "common.cuh"

namespace pa {

// One 16-byte chunk per thread per iteration.
//   k, v:  [num_tokens][hkv][row_chunks] int4 (row_chunks = head_dim * elem / 16)
//   kc, vc: [num_blocks][hkv][bs][row_chunks] int4
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(const int4* __restrict__ k, const int4* __restrict__ v,
                                                                const int64_t* __restrict__ slots, int4* __restrict__ kc,
                                                                int4* __restrict__ vc, int32_t num_tokens, int32_t hkv,
                                                                int32_t bs, int32_t row_chunks, int64_t num_slots) {
  const int64_t total = static_cast<int64_t>(num_tokens) * hkv * row_chunks;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int64_t row = i / row_chunks;
    const int32_t c = static_cast<int32_t>(i - row * row_chunks);
    const int64_t t = row / hkv;
    const int32_t h = static_cast<int32_t>(row - t * hkv);
    const int64_t slot = __ldg(slots + t);
    if (slot == -1) continue;
    if (slot < -1 || slot >= num_slots) {
      if (h == 0 && c == 0) record_error(PA_ERR_DEVICE_BOUNDS, slot);
      continue;
    }
    const int64_t blk = slot / bs;
    const int64_t off = slot - blk * bs;
    const int64_t dst = ((blk * hkv + h) * bs + off) * row_chunks + c;
    const int4 kx = __ldcs(k + i);
    const int4 vx = __ldcs(v + i);
    kc[dst] = kx;
    vc[dst] = vx;
  }
}

// 8-bit cache (CF: e4m3 or int8 codes): k, v rows are bf16 [num_tokens][hkv][D];
// each thread turns 16 bf16 inputs (two 16-byte loads) into one 16-byte store
// of codes.
//   row_chunks = D / 16 per (token, head) row
template <int CF>
__device__ __forceinline__ uint32_t quantize_code(float x, float scale) {
  if constexpr (CF == kCodeS8)
    return static_cast<uint8_t>(quantize_s8(x, scale));
  else
    return quantize_e4m3(x, scale);
}

template <int CF>
__global__ void __launch_bounds__(256) reshape_and_cache_q8_kernel(const uint4* __restrict__ k,
                                                                    const uint4* __restrict__ v,
                                                                    const int64_t* __restrict__ slots,
                                                                    int4* __restrict__ kc, int4* __restrict__ vc,
                                                                    int32_t num_tokens, int32_t hkv, int32_t bs,
                                                                    int32_t row_chunks, int64_t num_slots,
                                                                    float k_scale, float v_scale) {
  const int64_t total = static_cast<int64_t>(num_tokens) * hkv * row_chunks;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int64_t row = i / row_chunks;
    const int32_t c = static_cast<int32_t>(i - row * row_chunks);
    const int64_t t = row / hkv;
    const int32_t h = static_cast<int32_t>(row - t * hkv);
    const int64_t slot = __ldg(slots + t);
    if (slot == -1) continue;
    if (slot < -1 || slot >= num_slots) {
      if (h == 0 && c == 0) record_error(PA_ERR_DEVICE_BOUNDS, slot);
      continue;
    }
    const int64_t blk = slot / bs;
    const int64_t off = slot - blk * bs;
    const int64_t dst = ((blk * hkv + h) * bs + off) * row_chunks + c;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const uint4* src = (which == 0 ? k : v) + 2 * i;
      const float sc = which == 0 ? k_scale : v_scale;
      const uint4 a = __ldcs(src), b = __ldcs(src + 1);
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      uint32_t q[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t lo = w[2 * u], hi = w[2 * u + 1];
        q[u] = quantize_code<CF>(bf16lo(lo), sc) | (quantize_code<CF>(bf16hi(lo), sc) << 8) |
               (quantize_code<CF>(bf16lo(hi), sc) << 16) | (quantize_code<CF>(bf16hi(hi), sc) << 24);
      }
      (which == 0 ? kc : vc)[dst] = make_int4(q[0], q[1], q[2], q[3]);
    }
  }
}

// Grid: blocks_per_pair CTAs per pair, flattened. chunks = 16-byte chunks in
// one physical block of one tensor (hkv * bs * head_dim * elem / 16).
__global__ void __launch_bounds__(256) copy_blocks_kernel(int4* __restrict__ kc, int4* __restrict__ vc,
                                                          const int32_t* __restrict__ pairs, int32_t n_pairs,
                                                          int64_t chunks, int32_t blocks_per_pair, int64_t num_blocks) {
  const int32_t p = blockIdx.x / blocks_per_pair;
  const int32_t part = blockIdx.x - p * blocks_per_pair;
  if (p >= n_pairs) return;
  const int32_t src = __ldg(pairs + 2 * p);
  const int32_t dst = __ldg(pairs + 2 * p + 1);
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (part == 0 && threadIdx.x == 0) record_error(PA_ERR_DEVICE_BOUNDS, (src < 0 || src >= num_blocks) ? src : dst);
    return;
  }
  const int4* ks = kc + static_cast<int64_t>(src) * chunks;
  const int4* vs = vc + static_cast<int64_t>(src) * chunks;
  int4* kd = kc + static_cast<int64_t>(dst) * chunks;
  int4* vd = vc + static_cast<int64_t>(dst) * chunks;
  const int64_t stride = static_cast<int64_t>(blocks_per_pair) * blockDim.x;
  for (int64_t c = static_cast<int64_t>(part) * blockDim.x + threadIdx.x; c < chunks; c += stride) {
    const int4 a = ks[c];
    const int4 b = vs[c];
    kd[c] = a;
    vd[c] = b;
  }
}

// Swap whole blocks between the device pool and a host pool in pinned,
// device-mapped memory (same layout): dst[pair.y] = src[pair.x] for K and V.
// `src_nb` / `dst_nb` bound the ids on each side. Consecutive threads move
// consecutive 16-byte chunks, so the host side sees full-line PCIe transfers.
__global__ void __launch_bounds__(256) swap_blocks_kernel(const int4* __restrict__ sk, const int4* __restrict__ sv,
                                                          int4* __restrict__ dk, int4* __restrict__ dv,
                                                          const int32_t* __restrict__ pairs, int32_t n_pairs,
                                                          int64_t chunks, int32_t blocks_per_pair, int64_t src_nb,
                                                          int64_t dst_nb) {
  const int32_t p = blockIdx.x / blocks_per_pair;
  const int32_t part = blockIdx.x - p * blocks_per_pair;
  if (p >= n_pairs) return;
  const int32_t src = __ldg(pairs + 2 * p);
  const int32_t dst = __ldg(pairs + 2 * p + 1);
  if (src < 0 || src >= src_nb || dst < 0 || dst >= dst_nb) {
    if (part == 0 && threadIdx.x == 0) record_error(PA_ERR_DEVICE_BOUNDS, (src < 0 || src >= src_nb) ? src : dst);
    return;
  }
  const int4* ks = sk + static_cast<int64_t>(src) * chunks;
  const int4* vs = sv + static_cast<int64_t>(src) * chunks;
  int4* kd = dk + static_cast<int64_t>(dst) * chunks;
  int4* vd = dv + static_cast<int64_t>(dst) * chunks;
  const int64_t stride = static_cast<int64_t>(blocks_per_pair) * blockDim.x;
  for (int64_t c = static_cast<int64_t>(part) * blockDim.x + threadIdx.x; c < chunks; c += stride) {
    const int4 a = ks[c];
    const int4 b = vs[c];
    kd[c] = a;
    vd[c] = b;
  }
}

}  // namespace pa
