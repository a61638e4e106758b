// Pieces shared by the decode kernels: arguments, the chunk pipeline (TMA
// producer warp + consumer warps over full/empty mbarriers), the final merge
// of the consumer warps, and the partition merge kernel.
//
// P2 = "PagedAttention：操作系统级 KV 缓存虚拟内存管理", §4.1: the softmax is
// accumulated block by block with a running maximum and sum; the same algebra
// merges the warps of a CTA and the partitions of a sequence:
//   M = max_i m_i,  l = sum_i l_i 2^(m_i - M),  o = sum_i o_i 2^(m_i - M)
// (scores are kept in base 2: q is pre-scaled by scale * log2 e).
#pragma once

#include <type_traits>

#include "common.cuh"

namespace pa {

struct DecodeArgs {
  const void* q;
  const void* kc;
  const void* vc;
  const int32_t* tables;
  const int32_t* lens;
  float* out;
  float* ws_ml;   // [num_seqs][hq][parts_stride][2]  (m in log2 units, l)
  float* ws_o;    // [num_seqs][hq][parts_stride][D]
  int64_t num_blocks;
  int32_t num_seqs, hq, hkv, bs, max_blocks, max_ctx;
  int32_t part_tokens;  // > 0: partition size; 0: one partition per sequence
  int32_t max_parts;    // partitions of the longest sequence
  float scale_log2;     // scale * log2(e) (times the K scale of an fp8 cache)
  float v_scale = 1.f;  // V scale of an fp8 cache, applied to o before the merge
  // Persistent kernels: counters[0] hands out work items. Zeroed before every
  // launch.
  unsigned int* counters;
  int32_t n_items;      // hkv * num_seqs * max_parts
  // Shared-prefix (cascade) decode: this call covers tokens [starts[s], L_s)
  // only and always writes partials; prefix partials written by the cascade
  // prefix kernel sit after the suffix ones. Null / 0 / max_parts otherwise.
  const int32_t* starts;
  int32_t force_partials;
  int32_t parts_stride;  // partial slots per (sequence, query head) row
  int32_t prefix_part_tokens;  // tokens per prefix partial (cascade only)
  // Split sequences merged by the CTA that finishes last: each CTA counts its
  // arrival in counters[1 + s * hkv + g] (zeroed before the launch).
  int32_t fuse_merge = 0;
  // Cascade with unsplit suffixes: the suffix CTA of (s, g) merges its own
  // state with the sequence's prefix partials (written by the prefix pass,
  // earlier on the stream) and stores the final rows; a sequence with an empty
  // suffix still gets its partition-0 CTA for that merge.
  int32_t cascade_direct = 0;
  // Optional dispatch order: grid row y (or work item row) serves sequence
  // seq_order[y], a permutation of 0 .. num_seqs-1 (longest first puts the
  // long CTAs in the first waves). An entry out of range is recorded and that
  // row serves sequence y.
  const int32_t* seq_order = nullptr;
  // Host side: launch the decode kernel as the programmatic dependent of the
  // cascade prefix pass (it runs alongside that pass and waits for it before
  // folding in the prefix partials).
  int32_t after_prefix_pass = 0;
  // Fused KV append (pa_decode_append): the CTA, or persistent item, that
  // covers sequence s's last token first writes kv head g's new K and V rows
  // (k_new / v_new [num_seqs][hkv][D], bf16 for an 8-bit cache, else the
  // cache type) at slot_mapping[s] (-1: none), quantised with the cache's
  // k_scale / v_scale for an 8-bit cache. Null otherwise.
  const void* k_new = nullptr;
  const void* v_new = nullptr;
  const int64_t* slot_mapping = nullptr;
  int64_t num_slots = 0;  // num_blocks * bs
  float k_scale_store = 1.f, v_scale_store = 1.f;
};

// Sequence served by grid (or item) row y.
__device__ __forceinline__ int grid_seq(const DecodeArgs& a, int y, bool report) {
  if (!a.seq_order) return y;
  const int s = __ldg(a.seq_order + y);
  if (s < 0 || s >= a.num_seqs) {
    if (report) record_error(PA_ERR_DEVICE_BOUNDS, s);
    return y;
  }
  return s;
}

// First token a decode CTA covers for sequence s (the cascade suffix start).
__device__ __forceinline__ int32_t seq_start(const DecodeArgs& a, int32_t s, int32_t L) {
  if (!a.starts) return 0;
  int32_t st = __ldg(a.starts + s);
  return st < 0 ? 0 : (st > L ? L : st);
}

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
template <>
struct Elem<__nv_fp8_e4m3> {
  static constexpr int bytes = 1;
};
template <>
struct Elem<int8_t> {
  static constexpr int bytes = 1;
};

// Element type of q for a cache of element type T: an 8-bit cache is read
// with bf16 queries.
template <typename T>
struct QueryOf {
  using type = T;
};
template <>
struct QueryOf<__nv_fp8_e4m3> {
  using type = __nv_bfloat16;
};
template <>
struct QueryOf<int8_t> {
  using type = __nv_bfloat16;
};

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// Context length of sequence s, clamped to [0, max_ctx]; an out-of-range value
// is recorded (by the one thread that `report`s).
__device__ __forceinline__ int32_t load_len(const DecodeArgs& a, int32_t s, bool report) {
  int32_t L = __ldg(a.lens + s);
  if (L < 0 || L > a.max_ctx) {
    if (report) record_error(PA_ERR_DEVICE_BOUNDS, L);
    L = L < 0 ? 0 : a.max_ctx;
  }
  return L;
}

// The token range a CTA owns. Returns false if the CTA has nothing to do
// (after writing the zero row of an empty context).
struct Part {
  int32_t t0, t1, ntok, nparts;
  int32_t npre;  // cascade: prefix partials of this sequence (slots max_parts ..)
  bool last;     // covers the sequence's last token
};

template <int G, int D>
__device__ __forceinline__ bool cta_part(const DecodeArgs& a, int g, int s, int p, int tid, int nthreads, Part& pt) {
  const int32_t L = load_len(a, s, g == 0 && p == 0 && tid == 0);
  const int32_t st = seq_start(a, s, L);
  const int32_t span = L - st;
  const int32_t P = a.part_tokens > 0 ? a.part_tokens : (span > 0 ? span : 1);
  pt.t0 = st + p * P;
  pt.npre = 0;
  pt.last = false;
  if (a.starts && st > 0) {
    pt.npre = (st + a.prefix_part_tokens - 1) / a.prefix_part_tokens;
    pt.npre = min(pt.npre, a.parts_stride - a.max_parts);  // never past the prefix slots
  }
  if (L == 0 && !a.starts) {
    if (p == 0)
      for (int idx = tid; idx < G * D; idx += nthreads)
        a.out[(static_cast<int64_t>(s) * a.hq + g * G) * D + idx] = 0.f;
    return false;
  }
  if (a.cascade_direct && p == 0 && span == 0) {  // empty suffix: merge the prefix partials alone
    pt.t1 = pt.t0 = L;
    pt.ntok = 0;
    pt.nparts = 1;
    return true;
  }
  if (pt.t0 >= L) return false;
  pt.t1 = min(pt.t0 + P, L);
  pt.ntok = pt.t1 - pt.t0;
  pt.last = pt.t1 == L;
  pt.nparts = a.part_tokens > 0 ? (span + P - 1) / P : 1;
  return true;
}

// Fused KV append, by one warp (see DecodeArgs::k_new): load() reads kv head
// g's new K and V rows of sequence s into registers (at most two 16-byte
// pieces per lane at head_dim 128), write() stores them at the sequence's
// slot, publish() makes the stores visible to the async proxy, so that the
// bulk / tensor copies issued next (after a __syncwarp) read the new row.
// The producer loads at its start, writes once its first chunk's copies are
// issued, and publishes just before it issues the chunk that holds the slot
// (the CTA's last): the load and the store are then long complete and
// nothing waits for them. step() does that for chunk i of n.
template <typename T, int D>
struct AppendRow {
  static constexpr bool kCoded = Elem<T>::bytes == 1;
  // 16-byte pieces of the two cache rows (K then V); an 8-bit piece takes two
  // bf16 input pieces
  static constexpr int kPieces = kCoded ? 2 * (D / 16) : 2 * (D * Elem<T>::bytes / 16);
  static constexpr int kPerLane = (kPieces + 31) / 32;
  uint4 x[kPerLane][kCoded ? 2 : 1];
  int64_t row;  // cache row of the slot; -1: nothing to write

  __device__ __forceinline__ void load(const DecodeArgs& a, int s, int g, int lane) {
    const int64_t slot = __ldg(a.slot_mapping + s);
    row = -1;
    if (slot == -1) return;
    if (slot < 0 || slot >= a.num_slots) {
      if (lane == 0) record_error(PA_ERR_DEVICE_BOUNDS, slot);
      return;
    }
    const int64_t blk = slot / a.bs;
    row = (blk * a.hkv + g) * a.bs + (slot - blk * a.bs);
    const int64_t src_row = static_cast<int64_t>(s) * a.hkv + g;
    constexpr int CH = kPieces / 2;
#pragma unroll
    for (int u = 0; u < kPerLane; ++u) {
      const int i = lane + 32 * u;
      if (i < kPieces) {
        const int which = i / CH, c = i - which * CH;
        const uint4* src = static_cast<const uint4*>(which ? a.v_new : a.k_new);
        if constexpr (kCoded) {
          x[u][0] = __ldg(src + (src_row * CH + c) * 2);
          x[u][1] = __ldg(src + (src_row * CH + c) * 2 + 1);
        } else {
          x[u][0] = __ldg(src + src_row * CH + c);
        }
      }
    }
  }

  __device__ __forceinline__ void write(const DecodeArgs& a, int lane) {
    if (row < 0) return;
    // the cache pools are the caller's writable device memory (held const here for the readers)
    uint4* kc = static_cast<uint4*>(const_cast<void*>(a.kc));
    uint4* vc = static_cast<uint4*>(const_cast<void*>(a.vc));
    constexpr int CH = kPieces / 2;
#pragma unroll
    for (int u = 0; u < kPerLane; ++u) {
      const int i = lane + 32 * u;
      if (i < kPieces) {
        const int which = i / CH, c = i - which * CH;
        uint4 v = x[u][0];
        if constexpr (kCoded) {
          const float sc = which ? a.v_scale_store : a.k_scale_store;
          const uint32_t w[8] = {x[u][0].x, x[u][0].y, x[u][0].z, x[u][0].w,
                                 x[u][1].x, x[u][1].y, x[u][1].z, x[u][1].w};
          uint32_t q[4];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const float f[4] = {bf16lo(w[2 * e2]), bf16hi(w[2 * e2]), bf16lo(w[2 * e2 + 1]), bf16hi(w[2 * e2 + 1])};
            uint32_t b[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              if constexpr (std::is_same<T, int8_t>::value)
                b[e] = static_cast<uint8_t>(quantize_s8(f[e], sc));
              else
                b[e] = quantize_e4m3(f[e], sc);
            }
            q[e2] = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
          }
          v = make_uint4(q[0], q[1], q[2], q[3]);
        }
        (which ? vc : kc)[row * CH + c] = v;
      }
    }
  }

  __device__ __forceinline__ void publish() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

  // Before chunk i's copies (of n): the row goes out before the last chunk.
  __device__ __forceinline__ void before_chunk(const DecodeArgs& a, int i, int n, int lane) {
    if (i != n - 1) return;
    if (n == 1) write(a, lane);
    publish();
    __syncwarp();
  }
  // After chunk i's copies: the write, once the first chunk is on its way.
  __device__ __forceinline__ void after_chunk(const DecodeArgs& a, int i, int n, int lane) {
    if (i == 0 && n > 1) write(a, lane);
  }
};

// Work item -> (kv head g, sequence s, partition p), partition-major so that
// partition 0 of every sequence comes first.
__device__ __forceinline__ void item_coords(const DecodeArgs& a, int item, int& g, int& s, int& p) {
  const int per = a.hkv * a.num_seqs;
  p = item / per;
  const int r = item - p * per;
  s = r / a.hkv;
  g = r - s * a.hkv;
  s = grid_seq(a, s, g == 0);
}

// Named barrier over the four consumer warps (threads 0..127); the producer
// warp never joins it.
__device__ __forceinline__ void consumer_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Wait for a phase, giving up when the CTA's abort flag is raised by another
// warp or the wall-clock limit passes (then raising the flag itself).
__device__ __forceinline__ bool pipe_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t start = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - start > kWaitTimeoutNs) {
        record_error(PA_ERR_DEVICE_TIMEOUT, 0);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// Block ids of one table row, read ahead by the producer warp in windows of
// 32 entries (one per lane): the current window and the next are held in
// registers, so each chunk's ids (at most 8, block_size >= 8) come from
// shuffles, and the next window's load is in flight while the current one is
// used. Entries at or past `lim` are never read (they read as -1).
struct TableAhead {
  const int32_t* row;
  int32_t lim, w, cur, nxt;

  __device__ __forceinline__ int32_t fetch(int32_t win, int lane) const {
    const int32_t e = win * 32 + lane;
    return e < lim ? __ldg(row + e) : -1;
  }
  __device__ __forceinline__ void init(const int32_t* r, int32_t first_entry, int32_t lim_, int lane) {
    row = r;
    lim = lim_;
    w = first_entry >> 5;
    cur = fetch(w, lane);
    nxt = fetch(w + 1, lane);
  }
  // Entries e0 .. e0 + n - 1 (n <= 8, e0 never decreasing between calls):
  // lane u < n returns entry e0 + u, the other lanes -1. Whole warp.
  __device__ __forceinline__ int32_t get(int32_t e0, int n, int lane) {
    while ((e0 >> 5) > w) {
      cur = nxt;
      ++w;
      nxt = fetch(w + 1, lane);
    }
    int32_t mine = -1;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int32_t e = e0 + u;
      const int32_t v = __shfl_sync(0xffffffffu, (e >> 5) == w ? cur : nxt, e & 31);
      if (lane == u) mine = v;
    }
    return lane < n ? mine : -1;
  }
};

// Per-CTA pipeline state in shared memory: S stages, each with a "full"
// barrier (one producer arrival + the TMA byte count) and an "empty" barrier
// (one arrival per consumer warp).
template <int S>
struct PipeSmem {
  uint64_t full[S];
  uint64_t empty[S];
  int abort_flag;
};

template <int S>
__device__ __forceinline__ void pipe_init(PipeSmem<S>& ps, int consumer_warps) {
#pragma unroll
  for (int i = 0; i < S; ++i) {
    mbar_init(&ps.full[i], 1);
    mbar_init(&ps.empty[i], consumer_warps);
  }
  ps.abort_flag = 0;
  fence_mbar_init();
}

// Producer warp: for each chunk, wait until its stage is free, then let
// issue(i, stage) start the chunk's copies (issue arrives on full[stage] with
// the byte count). On abort, wait (bounded) for the copies already started.
template <int S, class Issue>
__device__ __forceinline__ void pipe_produce(PipeSmem<S>& ps, int nchunks, Issue issue) {
  int i = 0;
  for (; i < nchunks; ++i) {
    const int st = i % S;
    if (i >= S && !pipe_wait(&ps.empty[st], ((i / S) - 1) & 1, &ps.abort_flag)) break;
    issue(i, st);
  }
  if (ps.abort_flag) {
    // the latest phase of every stage that was filled must land before exit
    for (int j = (i > S ? i - S : 0); j < i; ++j) mbar_wait(&ps.full[j % S], (j / S) & 1);
  }
}

// Arrival of one partition of (sequence s, kv head g) whose partials are
// stored and fenced; true for the last of its nparts partitions.
__device__ __forceinline__ bool count_arrival(const DecodeArgs& a, int s, int g, int nparts) {
  const unsigned prev = atomicAdd(a.counters + 1 + static_cast<int64_t>(s) * a.hkv + g, 1u);
  __threadfence();
  return prev == static_cast<unsigned>(nparts - 1);
}

// The same log-sum-exp merge as decode_reduce_kernel, over the nparts
// partials of the G heads of kv head hq0 / G of sequence s, by threads
// tid = 0 .. nthreads-1, straight into out. The partials were written by other
// CTAs: read through L2 after the arrivals.
template <int G, int D>
__device__ __forceinline__ void merge_partials_to_out(const DecodeArgs& a, int s, int hq0, int nparts, int tid,
                                                      int nthreads) {
  __threadfence();
  for (int idx = tid; idx < G * D; idx += nthreads) {
    const int h = idx / D, d = idx - h * D;
    const int64_t row = static_cast<int64_t>(s) * a.hq + hq0 + h;
    const float* ml = a.ws_ml + row * a.parts_stride * 2;
    const float* po = a.ws_o + row * a.parts_stride * D + d;
    float M = -INFINITY;
    for (int q = 0; q < nparts; ++q) M = fmaxf(M, __ldcg(ml + 2 * q));
    float l = 0.f, o = 0.f;
    for (int q = 0; q < nparts; ++q) {
      const float f = exp2f(__ldcg(ml + 2 * q) - M);
      l = fmaf(__ldcg(ml + 2 * q + 1), f, l);
      o = fmaf(__ldcg(po + static_cast<int64_t>(q) * D), f, o);
    }
    a.out[row * D + d] = o / l;
  }
}

// Merge the consumer warps' (m, l, o) for the G heads of this CTA and store
// either the final row (one partition) or the partition's partials.
//   wm, wl: [NW][G];  wacc: [NW][G][D]
template <int G, int D, int NW>
__device__ __forceinline__ void merge_warps_and_store(const DecodeArgs& a, const float* wm, const float* wl,
                                                      const float* wacc, int s, int p, int hq0, int nparts, int npre,
                                                      int tid, int nthreads) {
  for (int idx = tid; idx < G * D; idx += nthreads) {
    const int h = idx / D, d = idx - h * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, wm[w * G + h]);
    float l = 0.f, o = 0.f;
    if (M != -INFINITY) {  // (an empty suffix has no state of its own)
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float f = exp2f(wm[w * G + h] - M);
        l = fmaf(wl[w * G + h], f, l);
        o = fmaf(wacc[(w * G + h) * D + d], f, o);
      }
    }
    const int64_t row = static_cast<int64_t>(s) * a.hq + hq0 + h;
    if (a.cascade_direct) {
      // fold in the prefix partials (written by the prefix pass: wait for it
      // when this grid was launched alongside it); each covers at least one
      // key, so its m is finite
      pdl_wait();
      const float* ml = a.ws_ml + (row * a.parts_stride + a.max_parts) * 2;
      const float* po = a.ws_o + (row * a.parts_stride + a.max_parts) * D + d;
      for (int q = 0; q < npre; ++q) {  // through L2: written by the other grid
        const float mq = __ldcg(ml + 2 * q);
        const float Mn = fmaxf(M, mq);
        const float f0 = exp2f(M - Mn), f1 = exp2f(mq - Mn);  // exp2(-inf) = 0 while M is -inf
        l = l * f0 + __ldcg(ml + 2 * q + 1) * f1;
        o = o * f0 + __ldcg(po + static_cast<int64_t>(q) * D) * f1;
        M = Mn;
      }
      a.out[row * D + d] = l > 0.f ? o / l : 0.f;  // an empty context gives a zero row
      continue;
    }
    if (nparts == 1 && !a.force_partials) {
      a.out[row * D + d] = o / l;
    } else {
      const int64_t prow = row * a.parts_stride + p;
      a.ws_o[prow * D + d] = o;
      if (d == 0) {
        a.ws_ml[prow * 2] = M;
        a.ws_ml[prow * 2 + 1] = l;
      }
    }
  }
  if (!a.fuse_merge || nparts == 1) return;
  // Merge in the last CTA of this (sequence, kv head).
  __shared__ int is_last;
  __threadfence();  // this thread's partials are visible device-wide ...
  __syncthreads();  // ... for every thread of the CTA, before the arrival counts
  if (tid == 0) is_last = count_arrival(a, s, hq0 / G, nparts);
  __syncthreads();
  if (is_last) merge_partials_to_out<G, D>(a, s, hq0, nparts, tid, nthreads);
}

// Merge the partitions of one (sequence, query head):
//   M = max_p m_p,  out = sum_p o_p 2^(m_p - M) / sum_p l_p 2^(m_p - M).
// A grid of a few CTAs per SM strides over the (sequence, query head) rows;
// 8 warps: warp w folds partitions w, w+8, ... with each lane owning D/32 dims
// (one coalesced row read per partition), then the warps are folded through
// shared memory. Sequences with one partition were written by the decode
// kernel and are skipped.
constexpr int kReduceWarps = 8;

template <int D>
__global__ void __launch_bounds__(32 * kReduceWarps) decode_reduce_kernel(const DecodeArgs a) {
  constexpr int VEC = D / 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __shared__ float red[kReduceWarps];
  __shared__ float wl[kReduceWarps];
  __shared__ float wo[kReduceWarps][D];
  const int64_t nrows = static_cast<int64_t>(a.num_seqs) * a.hq;
  // grid-stride over (sequence, query head) rows; rows of unsplit sequences are skipped
  for (int64_t row = blockIdx.x; row < nrows; row += gridDim.x) {
    const int s = static_cast<int>(row / a.hq);
    const int32_t L = load_len(a, s, false);
    const int32_t st = seq_start(a, s, L);
    const int32_t span = L - st;
    const int32_t P = a.part_tokens > 0 ? a.part_tokens : (span > 0 ? span : 1);
    const int32_t nsuf = span > 0 ? (span + P - 1) / P : 0;
    const int32_t npre = st > 0 ? (st + a.prefix_part_tokens - 1) / a.prefix_part_tokens : 0;
    if (!a.force_partials && nsuf <= 1) continue;  // written by the decode kernel; uniform across the CTA
    if (nsuf + npre == 0) {                        // empty context: zero row
      for (int d = tid; d < D; d += 32 * kReduceWarps) a.out[row * D + d] = 0.f;
      continue;
    }
    const int32_t nparts = nsuf + npre;
    const float* ml = a.ws_ml + row * a.parts_stride * 2;
    const float* o = a.ws_o + row * a.parts_stride * D;

    // slot of the i-th partial: suffix partials 0..nsuf-1, then prefix partials from max_parts on
    auto slot = [&](int i) { return i < nsuf ? i : a.max_parts + (i - nsuf); };
    float M = -INFINITY;
    for (int q = tid; q < nparts; q += 32 * kReduceWarps) M = fmaxf(M, ml[2 * slot(q)]);
    M = warp_max(M);
    if (lane == 0) red[warp] = M;
    __syncthreads();
    M = red[0];
#pragma unroll
    for (int w = 1; w < kReduceWarps; ++w) M = fmaxf(M, red[w]);

    float l = 0.f, acc[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
    // kUnroll partitions per warp per round: their loads are all in flight
    // before the first one is folded in (a long sequence has hundreds)
    constexpr int kUnroll = 4;
    for (int q0 = warp; q0 < nparts; q0 += kUnroll * kReduceWarps) {
      float mp[kUnroll], lp[kUnroll], x[kUnroll][VEC];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int q = q0 + u * kReduceWarps;
        mp[u] = -INFINITY;
        lp[u] = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) x[u][e] = 0.f;
        if (q < nparts) {
          const int sq = slot(q);
          mp[u] = ml[2 * sq];
          lp[u] = ml[2 * sq + 1];
          const float* src = o + static_cast<int64_t>(sq) * D + lane * VEC;
          if (VEC == 4) {
            const float4 v = *reinterpret_cast<const float4*>(src);
            x[u][0] = v.x, x[u][1] = v.y, x[u][2] = v.z, x[u][3] = v.w;
          } else {
#pragma unroll
            for (int e = 0; e < VEC; ++e) x[u][e] = src[e];
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const float f = exp2f(mp[u] - M);  // 0 for the empty slots of the last round
        l = fmaf(lp[u], f, l);
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] = fmaf(x[u][e], f, acc[e]);
      }
    }
    if (lane == 0) wl[warp] = l;
#pragma unroll
    for (int e = 0; e < VEC; ++e) wo[warp][lane * VEC + e] = acc[e];
    __syncthreads();
    for (int d = tid; d < D; d += 32 * kReduceWarps) {
      float num = 0.f, den = 0.f;
#pragma unroll
      for (int w = 0; w < kReduceWarps; ++w) {
        num += wo[w][d];
        den += wl[w];
      }
      a.out[row * D + d] = num / den;
    }
    __syncthreads();  // red / wl / wo are reused by the next row
  }
}

}  // namespace pa
