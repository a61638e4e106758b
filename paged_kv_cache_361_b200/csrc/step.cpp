// pa_step_host: one decode step from host memory, and its staging sizes.
//
// P2 = "PagedAttention：操作系统级 KV 缓存虚拟内存管理", §3.2.2 steps 1-4: the
// new token's K, V are computed by the model (the caller's host buffers); the
// block manager grows the tables (or copies a shared block, §3.4); the new K, V
// are written at their slots; attention runs over every block of the table.
// This file only orchestrates: block-manager calls on the host, one H2D copy of
// all step metadata (slots, CoW pairs, tables, lengths, each chunk's
// longest-first dispatch order) packed in pinned memory,
// the H2D copies of q/k/v, the device operations (copy-on-write copies, then the
// decode with the KV append fused, pa_decode_append), and the D2H copy of the
// output.
//
// A batch of at least kMinChunkRows sequences is cut into row chunks, each on
// a stream of its own (created once per device): chunk c's q/k/v copies, its
// append, its decode and its output copy form one chain, so the copy engines
// move chunk c+1's inputs and chunk c-1's output while chunk c computes, and the
// chunks' decodes share the SMs. The metadata copy and the copy-on-write block
// copies run first; every chunk waits for them. Small batches keep one chain
// on the caller's stream.
#include <cuda_runtime.h>

#include <algorithm>
#include <chrono>
#include <cstdint>
#include <mutex>
#include <vector>

#include "../../include/pagedattn.h"

namespace {

// Host-side phase times of the calling thread's last pa_step_host call.
thread_local pa_step_timing g_last_timing = {};

double us_since(std::chrono::steady_clock::time_point t0, std::chrono::steady_clock::time_point t1) {
  return std::chrono::duration<double, std::micro>(t1 - t0).count();
}

size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Row chunks of a batch (measured on the 64-sequence metric workload: one
// chain 0.281 ms per step, two 0.261 ms, four 0.274 ms: each chain costs host
// calls, ~15 us of enqueueing).
#ifndef PA_STEP_MAX_CHUNKS
#define PA_STEP_MAX_CHUNKS 2
#endif
constexpr int kMaxChunks = PA_STEP_MAX_CHUNKS;
constexpr int32_t kMinChunkRows = 8;

// Row chunks of a batch of n sequences: up to kMaxChunks of at least
// kMinChunkRows rows each.
int32_t num_chunks(int32_t n) { return std::max<int32_t>(1, std::min<int32_t>(kMaxChunks, n / kMinChunkRows)); }
int32_t chunk_rows(int32_t n, int32_t chunks) { return (n + chunks - 1) / chunks; }

struct StepLayout {
  int32_t cap;     // block-table columns
  int32_t chunks;  // row chunks (streams)
  // device regions (byte offsets into dev_staging)
  size_t q, k, v, out, meta, ws, dev_total, ws_bytes;  // ws_bytes: one chunk's workspace
  // metadata (same layout on host and device, starting at `meta`)
  size_t m_slots, m_pairs, m_tables, m_lens, m_order, meta_bytes;
};

bool make_layout(int32_t n, int32_t hq, const pa_cache* c, int32_t max_ctx, int32_t P, StepLayout& L) {
  if (!c || n < 0 || hq <= 0 || max_ctx < 0 || c->block_size <= 0 || c->head_dim <= 0 || c->num_kv_heads <= 0)
    return false;
  const size_t eb = c->dtype == PA_F32 ? 4 : 2;  // q, k, v inputs: bf16 for a bf16 or 8-bit cache
  const size_t N = static_cast<size_t>(n);
  L.cap = std::max<int32_t>(1, (max_ctx + c->block_size - 1) / c->block_size);
  L.chunks = num_chunks(n);
  L.m_slots = 0;
  L.m_pairs = up256(N * 8);
  L.m_tables = L.m_pairs + up256(N * 8);
  L.m_lens = L.m_tables + up256(N * L.cap * 4);
  L.m_order = L.m_lens + up256(N * 4);
  L.meta_bytes = L.m_order + up256(N * 4);
  L.q = 0;
  L.k = up256(N * hq * c->head_dim * eb);
  L.v = L.k + up256(N * c->num_kv_heads * c->head_dim * eb);
  L.out = L.v + up256(N * c->num_kv_heads * c->head_dim * eb);
  L.meta = L.out + up256(N * hq * c->head_dim * 4);
  L.ws = L.meta + L.meta_bytes;
  // each chunk decodes its rows with a workspace of its own (chunks run concurrently)
  // (chunks of `rows` rows, the last one possibly shorter)
  const int32_t rows = chunk_rows(n, L.chunks), last = n - (L.chunks - 1) * rows;
  const size_t ws = std::max(pa_decode_workspace_bytes(rows, hq, c->num_kv_heads, c->head_dim, max_ctx,
                                                       c->block_size, P),
                             pa_decode_workspace_bytes(last, hq, c->num_kv_heads, c->head_dim, max_ctx,
                                                       c->block_size, P));
  L.ws_bytes = up256(ws);
  L.dev_total = L.ws + L.ws_bytes * L.chunks;
  return true;
}

// Streams and events of the chunked step, created once per device.
struct StepStreams {
  cudaStream_t s[kMaxChunks];
  cudaEvent_t start, meta, done[kMaxChunks];
  bool ready = false;
};

StepStreams* step_streams() {
  static std::mutex mu;
  static StepStreams per_dev[64];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  StepStreams& S = per_dev[dev];
  if (!S.ready) {
    for (int i = 0; i < kMaxChunks; ++i)
      if (cudaStreamCreateWithFlags(&S.s[i], cudaStreamNonBlocking) != cudaSuccess ||
          cudaEventCreateWithFlags(&S.done[i], cudaEventDisableTiming) != cudaSuccess)
        return nullptr;
    if (cudaEventCreateWithFlags(&S.start, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&S.meta, cudaEventDisableTiming) != cudaSuccess)
      return nullptr;
    S.ready = true;
  }
  return &S;
}

}  // namespace

extern "C" pa_status pa_step_staging_bytes(int32_t n, int32_t num_q_heads, const pa_cache* cache,
                                           int32_t max_context_len, int32_t partition_tokens, size_t* dev_bytes,
                                           size_t* host_bytes) {
  StepLayout L;
  if (!dev_bytes || !host_bytes || partition_tokens < -1 ||
      !make_layout(n, num_q_heads, cache, max_context_len, partition_tokens, L))
    return PA_ERR_INVALID_ARG;
  *dev_bytes = L.dev_total;
  *host_bytes = L.meta_bytes;
  return PA_OK;
}

extern "C" pa_status pa_step_host(pa_bm* bm, const pa_cache* cache, int32_t n, const int64_t* seq_ids,
                                  int32_t num_q_heads, const void* q_host, const void* k_host, const void* v_host,
                                  float scale, float* out_host, int32_t partition_tokens, void* dev_staging,
                                  size_t dev_staging_bytes, void* host_staging, size_t host_staging_bytes,
                                  pa_stream stream) {
  using clock = std::chrono::steady_clock;
  const clock::time_point t_begin = clock::now();
  g_last_timing = pa_step_timing{};
  if (!bm || !cache || n < 0 || num_q_heads <= 0 || partition_tokens < -1) return PA_ERR_INVALID_ARG;
  if (n == 0) return PA_OK;
  if (!seq_ids || !q_host || !k_host || !v_host || !out_host || !dev_staging || !host_staging ||
      (reinterpret_cast<uintptr_t>(dev_staging) & 255) || (reinterpret_cast<uintptr_t>(host_staging) & 15))
    return PA_ERR_INVALID_ARG;

  // Lengths after the step; the ids must be distinct (one query row each).
  std::vector<int64_t> sorted(seq_ids, seq_ids + n);
  std::sort(sorted.begin(), sorted.end());
  if (std::adjacent_find(sorted.begin(), sorted.end()) != sorted.end()) return PA_ERR_INVALID_ARG;
  int64_t max_len = 0;
  for (int32_t i = 0; i < n; ++i) {
    int32_t nblk = 0;
    int64_t len = 0;
    pa_status st = pa_bm_block_table(bm, seq_ids[i], nullptr, 0, &nblk, &len);
    if (st != PA_OK) return st;
    max_len = std::max(max_len, len + 1);
  }
  if (max_len > INT32_MAX) return PA_ERR_UNSUPPORTED;
  StepLayout L;
  if (!make_layout(n, num_q_heads, cache, static_cast<int32_t>(max_len), partition_tokens, L))
    return PA_ERR_INVALID_ARG;
  if (L.dev_total > dev_staging_bytes || L.meta_bytes > host_staging_bytes) return PA_ERR_INVALID_ARG;
  StepStreams* SS = nullptr;
  if (L.chunks > 1 && !(SS = step_streams())) return PA_ERR_CUDA;

  // Host side of the step: slots (and CoW pairs), then the tables the decode reads.
  char* h = static_cast<char*>(host_staging);
  int32_t n_pairs = 0;
  pa_status st = pa_bm_append_slots(bm, n, seq_ids, reinterpret_cast<int64_t*>(h + L.m_slots),
                                    reinterpret_cast<int32_t*>(h + L.m_pairs), &n_pairs);
  if (st != PA_OK) return st;
  st = pa_bm_block_tables(bm, n, seq_ids, reinterpret_cast<int32_t*>(h + L.m_tables), L.cap, -1,
                          reinterpret_cast<int32_t*>(h + L.m_lens));
  if (st != PA_OK) return st;
  {
    // each chunk's decode dispatches its rows longest first (indices within the chunk)
    const int32_t* hl = reinterpret_cast<const int32_t*>(h + L.m_lens);
    int32_t* ho = reinterpret_cast<int32_t*>(h + L.m_order);
    const int32_t rows = chunk_rows(n, L.chunks);
    for (int32_t r0 = 0; r0 < n; r0 += rows) {
      const int32_t m = std::min(n, r0 + rows) - r0;
      for (int32_t i = 0; i < m; ++i) ho[r0 + i] = i;
      std::stable_sort(ho + r0, ho + r0 + m, [&](int32_t x, int32_t y) { return hl[r0 + x] > hl[r0 + y]; });
    }
  }
  const clock::time_point t_bm = clock::now();

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* d = static_cast<char*>(dev_staging);
  char* meta = d + L.meta;
  const size_t eb = cache->dtype == PA_F32 ? 4 : 2;
  const size_t q_row = static_cast<size_t>(num_q_heads) * cache->head_dim * eb;
  const size_t kv_row = static_cast<size_t>(cache->num_kv_heads) * cache->head_dim * eb;
  const size_t o_row = static_cast<size_t>(num_q_heads) * cache->head_dim * 4;
  const auto* slots = reinterpret_cast<const int64_t*>(meta + L.m_slots);
  const auto* tables = reinterpret_cast<const int32_t*>(meta + L.m_tables);
  const auto* lens = reinterpret_cast<const int32_t*>(meta + L.m_lens);
  const auto* order = reinterpret_cast<const int32_t*>(meta + L.m_order);
  float* out_dev = reinterpret_cast<float*>(d + L.out);

  // One chain: inputs of rows [r0, r1), their append and decode, their output back.
  auto chain = [&](cudaStream_t cs, int32_t r0, int32_t r1, char* ws) -> pa_status {
    const int32_t m = r1 - r0;
    if (cudaMemcpyAsync(d + L.q + r0 * q_row, static_cast<const char*>(q_host) + r0 * q_row, m * q_row,
                        cudaMemcpyHostToDevice, cs) != cudaSuccess ||
        cudaMemcpyAsync(d + L.k + r0 * kv_row, static_cast<const char*>(k_host) + r0 * kv_row, m * kv_row,
                        cudaMemcpyHostToDevice, cs) != cudaSuccess ||
        cudaMemcpyAsync(d + L.v + r0 * kv_row, static_cast<const char*>(v_host) + r0 * kv_row, m * kv_row,
                        cudaMemcpyHostToDevice, cs) != cudaSuccess)
      return PA_ERR_CUDA;
    // the KV append is done by the decode CTAs (one launch per chain)
    pa_status r = pa_decode_append(d + L.q + r0 * q_row, d + L.k + r0 * kv_row, d + L.v + r0 * kv_row, slots + r0, m,
                                   num_q_heads, cache, tables + static_cast<int64_t>(r0) * L.cap, L.cap, lens + r0,
                                   static_cast<int32_t>(max_len), order + r0, scale, out_dev + r0 * (o_row / 4),
                                   partition_tokens, L.ws_bytes ? ws : nullptr, L.ws_bytes, cs);
    if (r != PA_OK) return r;
    if (cudaMemcpyAsync(reinterpret_cast<char*>(out_host) + r0 * o_row, reinterpret_cast<char*>(out_dev) + r0 * o_row,
                        m * o_row, cudaMemcpyDeviceToHost, cs) != cudaSuccess)
      return PA_ERR_CUDA;
    return PA_OK;
  };

  if (L.chunks == 1) {
    if (cudaMemcpyAsync(meta, h, L.meta_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess) return PA_ERR_CUDA;
    if (n_pairs > 0) {
      st = pa_copy_blocks(cache, reinterpret_cast<const int32_t*>(meta + L.m_pairs), n_pairs, stream);
      if (st != PA_OK) return st;
    }
    const clock::time_point t_h2d = clock::now();
    st = chain(s, 0, n, d + L.ws);
    if (st != PA_OK) return st;
    const clock::time_point t_launch = clock::now();
    if (cudaStreamSynchronize(s) != cudaSuccess) return PA_ERR_CUDA;
    const clock::time_point t_end = clock::now();
    g_last_timing.block_manager_us = us_since(t_begin, t_bm);
    g_last_timing.metadata_enqueue_us = us_since(t_bm, t_h2d);
    g_last_timing.chains_enqueue_us = us_since(t_h2d, t_launch);
    g_last_timing.wait_us = us_since(t_launch, t_end);
    g_last_timing.total_us = us_since(t_begin, t_end);
    g_last_timing.chunks = 1;
    return PA_OK;
  }

  // Chunked: every chain starts after the caller's earlier work and after the
  // metadata and copy-on-write copies (chain 0's stream); the caller's stream
  // waits for every chain.
  cudaStream_t s0 = SS->s[0];
  if (cudaEventRecord(SS->start, s) != cudaSuccess) return PA_ERR_CUDA;
  for (int c = 0; c < L.chunks; ++c)
    if (cudaStreamWaitEvent(SS->s[c], SS->start, 0) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaMemcpyAsync(meta, h, L.meta_bytes, cudaMemcpyHostToDevice, s0) != cudaSuccess) return PA_ERR_CUDA;
  if (n_pairs > 0) {
    st = pa_copy_blocks(cache, reinterpret_cast<const int32_t*>(meta + L.m_pairs), n_pairs, s0);
    if (st != PA_OK) return st;
  }
  if (cudaEventRecord(SS->meta, s0) != cudaSuccess) return PA_ERR_CUDA;
  const clock::time_point t_h2d = clock::now();
  const int32_t rows = chunk_rows(n, L.chunks);
  for (int c = 0; c < L.chunks; ++c) {
    const int32_t r0 = c * rows, r1 = std::min(n, r0 + rows);
    if (r0 >= r1) break;
    if (c > 0 && cudaStreamWaitEvent(SS->s[c], SS->meta, 0) != cudaSuccess) return PA_ERR_CUDA;
    st = chain(SS->s[c], r0, r1, d + L.ws + c * L.ws_bytes);
    if (st != PA_OK) return st;
    if (cudaEventRecord(SS->done[c], SS->s[c]) != cudaSuccess || cudaStreamWaitEvent(s, SS->done[c], 0) != cudaSuccess)
      return PA_ERR_CUDA;
  }
  const clock::time_point t_launch = clock::now();
  if (cudaStreamSynchronize(s) != cudaSuccess) return PA_ERR_CUDA;
  const clock::time_point t_end = clock::now();
  g_last_timing.block_manager_us = us_since(t_begin, t_bm);
  g_last_timing.metadata_enqueue_us = us_since(t_bm, t_h2d);
  g_last_timing.chains_enqueue_us = us_since(t_h2d, t_launch);
  g_last_timing.wait_us = us_since(t_launch, t_end);
  g_last_timing.total_us = us_since(t_begin, t_end);
  g_last_timing.chunks = L.chunks;
  return PA_OK;
}

extern "C" pa_status pa_step_host_last_timing(pa_step_timing* out) {
  if (!out) return PA_ERR_INVALID_ARG;
  *out = g_last_timing;
  return PA_OK;
}
