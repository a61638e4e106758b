// pa_step_host: one decode step from host memory, and its staging sizes.
//
// P2 = "PagedAttention：操作系统级 KV 缓存虚拟内存管理", §3.2.2 steps 1-4: the
// new token's K, V are computed by the model (the caller's host buffers); the
// block manager grows the tables (or copies a shared block, §3.4); the new K, V
// are written at their slots; attention runs over every block of the table.
// This file only orchestrates: block-manager calls on the host, one H2D copy of
// all step metadata (slots, CoW pairs, tables, lengths) packed in pinned memory,
// the H2D copies of q/k/v, the three device operations, and the D2H copy of the
// output, all on one stream.
#include <cuda_runtime.h>

#include <algorithm>
#include <chrono>
#include <cstdint>
#include <vector>

#include "../../include/pagedattn.h"

namespace {

// Host-side phase times of the calling thread's last pa_step_host call.
thread_local pa_step_timing g_last_timing = {};

double us_since(std::chrono::steady_clock::time_point t0, std::chrono::steady_clock::time_point t1) {
  return std::chrono::duration<double, std::micro>(t1 - t0).count();
}

size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct StepLayout {
  int32_t cap;  // block-table columns
  // device regions (byte offsets into dev_staging)
  size_t q, k, v, out, meta, ws, dev_total, ws_bytes;
  // metadata (same layout on host and device, starting at `meta`)
  size_t m_slots, m_pairs, m_tables, m_lens, meta_bytes;
};

bool make_layout(int32_t n, int32_t hq, const pa_cache* c, int32_t max_ctx, int32_t P, StepLayout& L) {
  if (!c || n < 0 || hq <= 0 || max_ctx < 0 || c->block_size <= 0 || c->head_dim <= 0 || c->num_kv_heads <= 0)
    return false;
  const size_t eb = c->dtype == PA_F32 ? 4 : 2;  // q, k, v inputs: bf16 for a bf16 or fp8 cache
  const size_t N = static_cast<size_t>(n);
  L.cap = std::max<int32_t>(1, (max_ctx + c->block_size - 1) / c->block_size);
  L.m_slots = 0;
  L.m_pairs = up256(N * 8);
  L.m_tables = L.m_pairs + up256(N * 8);
  L.m_lens = L.m_tables + up256(N * L.cap * 4);
  L.meta_bytes = L.m_lens + up256(N * 4);
  L.q = 0;
  L.k = up256(N * hq * c->head_dim * eb);
  L.v = L.k + up256(N * c->num_kv_heads * c->head_dim * eb);
  L.out = L.v + up256(N * c->num_kv_heads * c->head_dim * eb);
  L.meta = L.out + up256(N * hq * c->head_dim * 4);
  L.ws = L.meta + L.meta_bytes;
  L.ws_bytes = pa_decode_workspace_bytes(n, hq, c->num_kv_heads, c->head_dim, max_ctx, c->block_size, P);
  L.dev_total = L.ws + up256(L.ws_bytes);
  return true;
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

  // Host side of the step: slots (and CoW pairs), then the tables the decode reads.
  char* h = static_cast<char*>(host_staging);
  int32_t n_pairs = 0;
  pa_status st = pa_bm_append_slots(bm, n, seq_ids, reinterpret_cast<int64_t*>(h + L.m_slots),
                                    reinterpret_cast<int32_t*>(h + L.m_pairs), &n_pairs);
  if (st != PA_OK) return st;
  st = pa_bm_block_tables(bm, n, seq_ids, reinterpret_cast<int32_t*>(h + L.m_tables), L.cap, -1,
                          reinterpret_cast<int32_t*>(h + L.m_lens));
  if (st != PA_OK) return st;
  const clock::time_point t_bm = clock::now();

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* d = static_cast<char*>(dev_staging);
  const size_t eb = cache->dtype == PA_F32 ? 4 : 2;
  const size_t qb = static_cast<size_t>(n) * num_q_heads * cache->head_dim * eb;
  const size_t kb = static_cast<size_t>(n) * cache->num_kv_heads * cache->head_dim * eb;
  if (cudaMemcpyAsync(d + L.meta, h, L.meta_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(d + L.q, q_host, qb, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(d + L.k, k_host, kb, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(d + L.v, v_host, kb, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return PA_ERR_CUDA;
  const clock::time_point t_h2d = clock::now();
  char* meta = d + L.meta;
  if (n_pairs > 0) {
    st = pa_copy_blocks(cache, reinterpret_cast<const int32_t*>(meta + L.m_pairs), n_pairs, stream);
    if (st != PA_OK) return st;
  }
  st = pa_reshape_and_cache(d + L.k, d + L.v, reinterpret_cast<const int64_t*>(meta + L.m_slots), n, cache, stream);
  if (st != PA_OK) return st;
  float* out_dev = reinterpret_cast<float*>(d + L.out);
  st = pa_decode(d + L.q, n, num_q_heads, cache, reinterpret_cast<const int32_t*>(meta + L.m_tables), L.cap,
                 reinterpret_cast<const int32_t*>(meta + L.m_lens), static_cast<int32_t>(max_len), scale, out_dev,
                 partition_tokens, L.ws_bytes ? d + L.ws : nullptr, L.ws_bytes, stream);
  if (st != PA_OK) return st;
  const clock::time_point t_launch = clock::now();
  const size_t ob = static_cast<size_t>(n) * num_q_heads * cache->head_dim * 4;
  if (cudaMemcpyAsync(out_host, out_dev, ob, cudaMemcpyDeviceToHost, s) != cudaSuccess) return PA_ERR_CUDA;
  const clock::time_point t_d2h = clock::now();
  if (cudaStreamSynchronize(s) != cudaSuccess) return PA_ERR_CUDA;
  const clock::time_point t_end = clock::now();
  g_last_timing.block_manager_us = us_since(t_begin, t_bm);
  g_last_timing.h2d_enqueue_us = us_since(t_bm, t_h2d);
  g_last_timing.launch_us = us_since(t_h2d, t_launch);
  g_last_timing.d2h_enqueue_us = us_since(t_launch, t_d2h);
  g_last_timing.wait_us = us_since(t_d2h, t_end);
  g_last_timing.total_us = us_since(t_begin, t_end);
  return PA_OK;
}

extern "C" pa_status pa_step_host_last_timing(pa_step_timing* out) {
  if (!out) return PA_ERR_INVALID_ARG;
  *out = g_last_timing;
  return PA_OK;
}
