// C-ABI entry points of libpagedattn: argument checks, kernel selection and
// launches. The declarations and their contracts are in include/pagedattn.h.
#include <cmath>
#include <cstdint>
#include <mutex>
#include <type_traits>
#include <utility>
#include <vector>

#include <cudaTypedefs.h>

#include "cache_ops.cuh"
#include "decode_f8.cuh"
#include "decode_mma.cuh"
#include "decode_simt.cuh"
#include "prefill_mma.cuh"
#include "prefill_tc.cuh"

namespace {

using namespace pa;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool pow2_block(int32_t bs) { return bs == 1 || bs == 2 || bs == 4 || bs == 8 || bs == 16 || bs == 32; }
bool is_8bit(int32_t dtype) { return dtype == PA_FP8_E4M3 || dtype == PA_INT8; }
int elem_bytes(int32_t dtype) { return is_8bit(dtype) ? 1 : (dtype == PA_BF16 ? 2 : 4); }

pa_status check_cache(const pa_cache* c) {
  if (!c || !c->k || !c->v || !aligned16(c->k) || !aligned16(c->v)) return PA_ERR_INVALID_ARG;
  if (c->num_blocks <= 0 || c->num_blocks > INT32_MAX || c->num_kv_heads <= 0) return PA_ERR_INVALID_ARG;
  if (c->head_dim != 64 && c->head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (!pow2_block(c->block_size)) return PA_ERR_UNSUPPORTED;
  if (c->dtype != PA_F32 && c->dtype != PA_BF16 && !is_8bit(c->dtype)) return PA_ERR_UNSUPPORTED;
  if (is_8bit(c->dtype) && !(std::isfinite(c->k_scale) && c->k_scale > 0.f && std::isfinite(c->v_scale) &&
                             c->v_scale > 0.f))
    return PA_ERR_INVALID_ARG;
  // slots must fit in int64 and block ids in int32 (checked above)
  return PA_OK;
}

pa_status launched() { return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA; }

// Launches kern on st. With after_prev the launch carries the
// programmatic-stream-serialization attribute: the grid may start once the
// previous grid on the stream has called pdl_launch_dependents(), and it must
// call pdl_wait() before it reads anything that grid writes.
template <typename... KArgs, typename... Args>
pa_status launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool after_prev,
                        Args&&... args) {
  if (!after_prev) {
    kern<<<grid, block, smem, st>>>(std::forward<Args>(args)...);
    return launched();
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// Partition size for partition_tokens = -1. Measured on a B200 with the
// decode kernels here: unsplit CTAs win while there are enough (sequence, kv
// head) units to fill the GPU and no unit is long; long units are cut into
// 1024 tokens (many units) or 2048 tokens (fewer units) to balance the SMs;
// with very few units the sequences are cut so that about 600 CTAs exist.
// When the CTAs are dispatched longest first (ordered), the waves balance
// themselves: with at least 1024 units and contexts up to 8192 tokens no
// split pays (continuous batching, 2048 units up to 4097 tokens: 0.1398 ms
// unsplit against 0.1684 ms at 1024-token partitions).
int32_t resolve_partition(int32_t num_seqs, int32_t hkv, int32_t max_ctx, int32_t bs, int32_t requested,
                          bool ordered = false) {
  if (requested >= 0) return requested;
  const int64_t units = static_cast<int64_t>(num_seqs) * hkv;
  int64_t P;
  if (units >= 256 && max_ctx <= 2560) return 0;
  if (ordered && units >= 1024 && max_ctx <= 8192) return 0;
  if (units >= 1024) {
    P = 1024;
  } else if (units >= 256) {
    P = 2048;
  } else {
    const int64_t parts = (600 + units - 1) / (units > 0 ? units : 1);
    P = (max_ctx + parts - 1) / parts;
    P = P < 512 ? 512 : (P > 2048 ? 2048 : P);
  }
  P = (P + bs - 1) / bs * bs;
  return P >= max_ctx ? 0 : static_cast<int32_t>(P);
}

// Split decodes with fewer partitions than this merge in their last CTA.
constexpr int32_t kFuseMergeMaxParts = 8;

int32_t num_parts(int32_t max_ctx, int32_t P) {
  if (P <= 0 || max_ctx <= 0) return 1;
  return (max_ctx + P - 1) / P;
}

// Workspace: [work counters (1 + num_seqs * hkv) x u32, 256-aligned]
//            [split partials (m, l): num_seqs * hq * parts x 2 floats, 256-aligned]
//            [split partials o: num_seqs * hq * parts x D floats]
size_t counters_bytes(int32_t num_seqs, int32_t hkv) {
  return (static_cast<size_t>(1 + static_cast<int64_t>(num_seqs) * hkv) * 4 + 255) / 256 * 256;
}
size_t ml_bytes(int32_t num_seqs, int32_t hq, int32_t max_parts) {
  return (static_cast<size_t>(num_seqs) * hq * max_parts * 2 * sizeof(float) + 255) / 256 * 256;
}
size_t ws_bytes(int32_t num_seqs, int32_t hq, int32_t hkv, int32_t D, int32_t max_parts) {
  size_t b = counters_bytes(num_seqs, hkv);
  if (max_parts > 1) b += ml_bytes(num_seqs, hq, max_parts) + static_cast<size_t>(num_seqs) * hq * max_parts * D * 4;
  return b;
}

int device_sm_count() {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

// Sets a kernel's dynamic shared-memory limit (and the max-shared carveout)
// once per (kernel, device): the attributes persist for the process, and the
// per-token host path should not pay for the calls on every launch.
bool smem_attrs(const void* kern, int bytes, bool max_carveout) {
  static std::mutex mu;
  static std::vector<std::pair<std::pair<const void*, int>, int>> done;  // ((kernel, device), bytes)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lock(mu);
  for (const auto& e : done)
    if (e.first.first == kern && e.first.second == dev && e.second >= bytes) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  if (max_carveout &&
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared) !=
          cudaSuccess)
    return false;
  done.push_back({{kern, dev}, bytes});
  return true;
}

template <typename T, int D, int G>
pa_status launch_simt(const DecodeArgs& a, dim3 grid, cudaStream_t st) {
  using Cfg = SimtCfg<T, D>;
  auto kern = decode_simt_kernel<T, D, G>;
  if (!smem_attrs(reinterpret_cast<const void*>(kern), Cfg::kSmemBytes, true)) return PA_ERR_CUDA;
  return launch_kernel(kern, grid, dim3(Cfg::kThreads), Cfg::kSmemBytes, st, a.after_prefix_pass != 0, a);
}

template <typename T, int D>
pa_status dispatch_g(const DecodeArgs& a, int G, dim3 grid, cudaStream_t st) {
  switch (G) {
    case 1: return launch_simt<T, D, 1>(a, grid, st);
    case 2: return launch_simt<T, D, 2>(a, grid, st);
    case 4: return launch_simt<T, D, 4>(a, grid, st);
    case 8: return launch_simt<T, D, 8>(a, grid, st);
    default: return PA_ERR_UNSUPPORTED;
  }
}

// cuTensorMapEncodeTiled, reached through the runtime so that the library
// needs no link-time dependency on the driver library.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// The pool viewed as rows of head_dim bf16 (row = (block * Hkv + head) * bs +
// offset), read in [bs x 64] boxes with the 128-byte swizzle.
bool encode_rows(CUtensorMap* map, void* base, uint64_t rows, int D, int bs) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), rows};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(bs)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A bf16 pool with head_dim 128 for the grouped-head decode: one copy per
// (block, head) tile. Dimensions (64 elements, pool rows, 2 halves) with byte
// strides (256 per row, 128 per half) and a box of (64, bs, 2): the copy
// lands as [half][row][128 bytes] with the 128-byte swizzle, as the two 2-D
// column boxes would, in one request instead of two.
bool encode_rows_halves(CUtensorMap* map, void* base, uint64_t rows, int bs) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[3] = {64, rows, 2};
  const cuuint64_t strides[2] = {256, 128};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(bs), 2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The prefill output [tokens][heads][head_dim] fp32 as a 3-D map for TMA
// stores of [128 / G tokens x G heads x 32 columns] boxes (one query tile's O
// in 32-column slices) with the 128-byte swizzle. `tokens` bounds the rows the
// kernel stores (only tiles whose rows are all inside their sequence).
bool encode_out_tiles(CUtensorMap* map, void* base, uint64_t tokens, int hq, int D, int G) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(hq), tokens};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 4, static_cast<cuuint64_t>(hq) * D * 4};
  const cuuint32_t box[3] = {32, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(128 / G)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The prefill queries [tokens][heads][head_dim] bf16 as a 3-D map for TMA
// loads of [128 / G tokens x G heads x 64 dims] boxes (one 64-dim half of a
// query tile) with the 128-byte swizzle. The kernel loads only tiles whose
// rows are all inside their sequence, so every row it reads exists.
bool encode_q_tiles(CUtensorMap* map, void* base, uint64_t tokens, int hq, int D, int G) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(hq), tokens};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(hq) * D * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(128 / G)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// An e4m3 pool viewed as rows of head_dim bytes, read in [bs x head_dim] boxes
// with the 128-byte (head_dim 128) or 64-byte (head_dim 64) swizzle.
bool encode_rows_u8(CUtensorMap* map, void* base, uint64_t rows, int D, int bs) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), rows};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(D), static_cast<cuuint32_t>(bs)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor-core decode over an 8-bit cache (block_size >= 8, pool rows addressable by the TMA).
bool f8_mma_eligible(const pa_cache* c) {
  return is_8bit(c->dtype) && c->block_size >= 8 &&
         static_cast<int64_t>(c->num_blocks) * c->num_kv_heads * c->block_size <= INT32_MAX;
}

template <int D, int G, int CF>
pa_status launch_f8(const DecodeArgs& a, const pa_cache* c, dim3 grid, cudaStream_t st) {
  using Cfg = F8Cfg<D>;
  CUtensorMap tk, tv;
  const uint64_t rows = static_cast<uint64_t>(c->num_blocks) * c->num_kv_heads * c->block_size;
  if (!encode_rows_u8(&tk, c->k, rows, D, c->block_size) || !encode_rows_u8(&tv, c->v, rows, D, c->block_size))
    return PA_ERR_CUDA;
  auto kern = decode_f8_kernel<D, G, CF>;
  if (!smem_attrs(reinterpret_cast<const void*>(kern), Cfg::kSmemBytes, true)) return PA_ERR_CUDA;
  return launch_kernel(kern, grid, dim3(Cfg::kThreads), Cfg::kSmemBytes, st, a.after_prefix_pass != 0, tk, tv, a);
}

template <int D, int CF>
pa_status dispatch_f8_cf(const DecodeArgs& a, const pa_cache* c, int G, dim3 grid, cudaStream_t st) {
  switch (G) {
    case 1: return launch_f8<D, 1, CF>(a, c, grid, st);
    case 2: return launch_f8<D, 2, CF>(a, c, grid, st);
    case 4: return launch_f8<D, 4, CF>(a, c, grid, st);
    case 8: return launch_f8<D, 8, CF>(a, c, grid, st);
    default: return PA_ERR_UNSUPPORTED;
  }
}

template <int D>
pa_status dispatch_f8(const DecodeArgs& a, const pa_cache* c, int G, dim3 grid, cudaStream_t st) {
  return c->dtype == PA_INT8 ? dispatch_f8_cf<D, kCodeS8>(a, c, G, grid, st)
                             : dispatch_f8_cf<D, kCodeE4M3>(a, c, G, grid, st);
}

template <int D, int G>
pa_status launch_mma(const DecodeArgs& a, const pa_cache* c, bool persistent, cudaStream_t st) {
  using Cfg = MmaCfg<D>;
  CUtensorMap tk, tv;
  const uint64_t rows = static_cast<uint64_t>(c->num_blocks) * c->num_kv_heads * c->block_size;
  const bool ok = D == 128 ? encode_rows_halves(&tk, c->k, rows, c->block_size) &&
                                 encode_rows_halves(&tv, c->v, rows, c->block_size)
                           : encode_rows(&tk, c->k, rows, D, c->block_size) &&
                                 encode_rows(&tv, c->v, rows, D, c->block_size);
  if (!ok) return PA_ERR_CUDA;
  if (!persistent) {
    auto kern = decode_mma_kernel<D, G>;
    if (!smem_attrs(reinterpret_cast<const void*>(kern), Cfg::kSmemBytes, true)) return PA_ERR_CUDA;
    return launch_kernel(kern, dim3(a.hkv, a.num_seqs, a.max_parts), dim3(Cfg::kThreads), Cfg::kSmemBytes, st,
                         a.after_prefix_pass != 0, tk, tv, a);
  }
  auto kern = decode_mma_persistent_kernel<D, G>;
  static int occ[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return PA_ERR_CUDA;
  if (!occ[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kPersistSmemBytes) !=
            cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared) !=
            cudaSuccess)
      return PA_ERR_CUDA;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, Cfg::kThreads, Cfg::kPersistSmemBytes) !=
            cudaSuccess ||
        n < 1)
      return PA_ERR_CUDA;
    occ[dev] = n;
  }
  // one CTA per resident slot; work items handed out by counters[0]
  if (cudaMemsetAsync(a.counters, 0, counters_bytes(a.num_seqs, a.hkv), st) != cudaSuccess) return PA_ERR_CUDA;
  const int64_t slots = static_cast<int64_t>(occ[dev]) * device_sm_count();
  const unsigned grid = static_cast<unsigned>(a.n_items < slots ? a.n_items : slots);
  kern<<<grid, Cfg::kThreads, Cfg::kPersistSmemBytes, st>>>(tk, tv, a);
  return launched();
}

// Tensor-core path: bf16 cache, a group of 4 or 8 query heads, blocks of at
// least 8 tokens (a [bs x 64] box is then a whole number of 1 KB swizzle
// atoms), and pool rows addressable by a 32-bit TMA coordinate.
bool mma_eligible(const pa_cache* c, int G) {
  return c->dtype == PA_BF16 && (G == 4 || G == 8) && c->block_size >= 8 &&
         static_cast<int64_t>(c->num_blocks) * c->num_kv_heads * c->block_size <= INT32_MAX;
}

// Persistent CTAs pay off when long sequences are cut into many short, equal
// partitions (measured on a B200: 512-token partitions of 32k-131k contexts
// gain ~12 %); with few or unequal work items one CTA per item balances better.
// (The continuous-batching trace, 1024-token partitions of 256 sequences,
// gained 6 % over one CTA per item.)
#ifndef PA_MMA_PERSIST_MIN_PARTS
#define PA_MMA_PERSIST_MIN_PARTS 2
#endif
bool mma_persistent(const DecodeArgs& a) {
  return a.part_tokens > 0 && a.part_tokens <= 1024 && a.max_parts >= PA_MMA_PERSIST_MIN_PARTS;
}

pa_status dispatch_mma(const DecodeArgs& a, const pa_cache* c, int G, cudaStream_t st) {
  const bool persistent = mma_persistent(a);
  if (c->head_dim == 128)
    return G == 8 ? launch_mma<128, 8>(a, c, persistent, st) : launch_mma<128, 4>(a, c, persistent, st);
  return G == 8 ? launch_mma<64, 8>(a, c, persistent, st) : launch_mma<64, 4>(a, c, persistent, st);
}

// One thread waits on an mbarrier that nothing will complete: exercises the
// bounded-wait path that every pipelined kernel uses.
__global__ void selftest_wait_kernel(uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  mbar_init(&bar, 1);
  fence_mbar_init();
  mbar_wait(&bar, 0, timeout_ns);
}

template <int D>
pa_status launch_reduce(const DecodeArgs& a, cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(a.num_seqs) * a.hq;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 8;
  decode_reduce_kernel<D><<<static_cast<unsigned>(rows < cap ? rows : cap), 32 * kReduceWarps, 0, st>>>(a);
  return launched();
}

}  // namespace

extern "C" {

const char* pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case PA_ERR_NO_FREE_BLOCKS: return "no free blocks";
    case PA_ERR_UNKNOWN_SEQ: return "unknown sequence";
    case PA_ERR_SEQ_EXISTS: return "sequence already exists";
    case PA_ERR_CUDA: return "CUDA error";
    case PA_ERR_DEVICE_BOUNDS: return "device index out of bounds";
    case PA_ERR_DEVICE_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

int32_t pa_version(void) { return 1; }

pa_status pa_reshape_and_cache(const void* k, const void* v, const int64_t* slot_mapping, int32_t num_tokens,
                               const pa_cache* cache, pa_stream stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_tokens < 0) return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !slot_mapping || !aligned16(k) || !aligned16(v) || (reinterpret_cast<uintptr_t>(slot_mapping) & 7))
    return PA_ERR_INVALID_ARG;
  const int32_t row_chunks = cache->head_dim * elem_bytes(cache->dtype) / 16;
  const int64_t total = static_cast<int64_t>(num_tokens) * cache->num_kv_heads * row_chunks;
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 64) blocks = 148 * 64;  // grid-stride beyond this
  if (is_8bit(cache->dtype)) {
    auto kern = cache->dtype == PA_INT8 ? reshape_and_cache_q8_kernel<kCodeS8> : reshape_and_cache_q8_kernel<kCodeE4M3>;
    kern<<<static_cast<unsigned>(blocks), threads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(k), static_cast<const uint4*>(v), slot_mapping, static_cast<int4*>(cache->k),
        static_cast<int4*>(cache->v), num_tokens, cache->num_kv_heads, cache->block_size, row_chunks,
        cache->num_blocks * cache->block_size, cache->k_scale, cache->v_scale);
    return launched();
  }
  reshape_and_cache_kernel<<<static_cast<unsigned>(blocks), threads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const int4*>(k), static_cast<const int4*>(v), slot_mapping, static_cast<int4*>(cache->k),
      static_cast<int4*>(cache->v), num_tokens, cache->num_kv_heads, cache->block_size, row_chunks,
      cache->num_blocks * cache->block_size);
  return launched();
}

pa_status pa_copy_blocks(const pa_cache* cache, const int32_t* src_dst_pairs, int32_t n_pairs, pa_stream stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (n_pairs < 0) return PA_ERR_INVALID_ARG;
  if (n_pairs == 0) return PA_OK;
  if (!src_dst_pairs || (reinterpret_cast<uintptr_t>(src_dst_pairs) & 7)) return PA_ERR_INVALID_ARG;
  const int64_t chunks = static_cast<int64_t>(cache->num_kv_heads) * cache->block_size * cache->head_dim *
                         elem_bytes(cache->dtype) / 16;
  const int threads = 256;
  int64_t bpp = (chunks + threads * 4 - 1) / (threads * 4);  // ~4 vectors per thread per tensor
  if (bpp < 1) bpp = 1;
  const int64_t grid = bpp * n_pairs;
  if (grid > INT32_MAX) return PA_ERR_UNSUPPORTED;
  copy_blocks_kernel<<<static_cast<unsigned>(grid), threads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<int4*>(cache->k), static_cast<int4*>(cache->v), src_dst_pairs, n_pairs, chunks,
      static_cast<int32_t>(bpp), cache->num_blocks);
  return launched();
}

pa_status pa_swap_blocks(const pa_cache* cache, void* host_k, void* host_v, int64_t host_num_blocks,
                         const int32_t* pairs, int32_t n_pairs, int32_t to_host, pa_stream stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (n_pairs < 0 || host_num_blocks <= 0 || host_num_blocks > INT32_MAX) return PA_ERR_INVALID_ARG;
  if (n_pairs == 0) return PA_OK;
  if (!host_k || !host_v || !pairs || !aligned16(host_k) || !aligned16(host_v) ||
      (reinterpret_cast<uintptr_t>(pairs) & 7))
    return PA_ERR_INVALID_ARG;
  // The host pools must be pinned and mapped into the device's address space:
  // a kernel touching pageable memory would fault.
  void* dk_host = nullptr;
  void* dv_host = nullptr;
  for (int i = 0; i < 2; ++i) {
    void* hp = i == 0 ? host_k : host_v;
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, hp) != cudaSuccess) {
      cudaGetLastError();
      return PA_ERR_INVALID_ARG;
    }
    if (attr.type != cudaMemoryTypeHost || !attr.devicePointer) return PA_ERR_INVALID_ARG;
    (i == 0 ? dk_host : dv_host) = attr.devicePointer;
  }
  const int64_t chunks = static_cast<int64_t>(cache->num_kv_heads) * cache->block_size * cache->head_dim *
                         elem_bytes(cache->dtype) / 16;
  const int threads = 256;
  int64_t bpp = (chunks + threads * 2 - 1) / (threads * 2);
  if (bpp < 1) bpp = 1;
  const int64_t grid = bpp * n_pairs;
  if (grid > INT32_MAX) return PA_ERR_UNSUPPORTED;
  const int4* sk = static_cast<const int4*>(to_host ? cache->k : dk_host);
  const int4* sv = static_cast<const int4*>(to_host ? cache->v : dv_host);
  int4* dk = static_cast<int4*>(to_host ? dk_host : cache->k);
  int4* dv = static_cast<int4*>(to_host ? dv_host : cache->v);
  swap_blocks_kernel<<<static_cast<unsigned>(grid), threads, 0, static_cast<cudaStream_t>(stream)>>>(
      sk, sv, dk, dv, pairs, n_pairs, chunks, static_cast<int32_t>(bpp), to_host ? cache->num_blocks : host_num_blocks,
      to_host ? host_num_blocks : cache->num_blocks);
  return launched();
}

pa_status pa_swap_blocks_copy(const pa_cache* cache, void* host_k, void* host_v, int64_t host_num_blocks,
                              const int32_t* host_pairs, int32_t n_pairs, int32_t to_host, pa_stream stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (n_pairs < 0 || host_num_blocks <= 0 || host_num_blocks > INT32_MAX) return PA_ERR_INVALID_ARG;
  if (n_pairs == 0) return PA_OK;
  if (!host_k || !host_v || !host_pairs) return PA_ERR_INVALID_ARG;
  for (int i = 0; i < 2; ++i) {
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, i == 0 ? host_k : host_v) != cudaSuccess) {
      cudaGetLastError();
      return PA_ERR_INVALID_ARG;
    }
    if (attr.type != cudaMemoryTypeHost) return PA_ERR_INVALID_ARG;  // pinned only: async copies
  }
  const int64_t src_nb = to_host ? cache->num_blocks : host_num_blocks;
  const int64_t dst_nb = to_host ? host_num_blocks : cache->num_blocks;
  for (int32_t p = 0; p < n_pairs; ++p) {
    const int32_t a = host_pairs[2 * p], b = host_pairs[2 * p + 1];
    if (a < 0 || a >= src_nb || b < 0 || b >= dst_nb) return PA_ERR_INVALID_ARG;
  }
  const size_t blk = static_cast<size_t>(cache->num_kv_heads) * cache->block_size * cache->head_dim *
                     elem_bytes(cache->dtype);
  char* sk = static_cast<char*>(to_host ? cache->k : host_k);
  char* sv = static_cast<char*>(to_host ? cache->v : host_v);
  char* dk = static_cast<char*>(to_host ? host_k : cache->k);
  char* dv = static_cast<char*>(to_host ? host_v : cache->v);
  const cudaMemcpyKind kind = to_host ? cudaMemcpyDeviceToHost : cudaMemcpyHostToDevice;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int32_t p = 0; p < n_pairs;) {
    int32_t q = p + 1;  // extend the run while both ids advance by one
    while (q < n_pairs && host_pairs[2 * q] == host_pairs[2 * q - 2] + 1 &&
           host_pairs[2 * q + 1] == host_pairs[2 * q - 1] + 1)
      ++q;
    const size_t off_s = static_cast<size_t>(host_pairs[2 * p]) * blk;
    const size_t off_d = static_cast<size_t>(host_pairs[2 * p + 1]) * blk;
    const size_t bytes = static_cast<size_t>(q - p) * blk;
    if (cudaMemcpyAsync(dk + off_d, sk + off_s, bytes, kind, s) != cudaSuccess ||
        cudaMemcpyAsync(dv + off_d, sv + off_s, bytes, kind, s) != cudaSuccess)
      return PA_ERR_CUDA;
    p = q;
  }
  return PA_OK;
}

pa_status pa_prefill(const void* q, int32_t num_seqs, const int32_t* cu_q_lens, int32_t max_q_len, int32_t num_q_heads,
                     const pa_cache* cache, const int32_t* block_tables, int32_t max_blocks_per_seq,
                     const int32_t* context_lens, int32_t max_context_len, float scale, float* out, pa_stream stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || max_q_len < 0 || num_q_heads <= 0 || max_blocks_per_seq <= 0 || max_context_len < 0)
    return PA_ERR_INVALID_ARG;
  if (num_q_heads % cache->num_kv_heads) return PA_ERR_INVALID_ARG;
  const int G = num_q_heads / cache->num_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
  if ((cache->dtype != PA_BF16 && !is_8bit(cache->dtype)) || cache->block_size < 8) return PA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(cache->num_blocks) * cache->num_kv_heads * cache->block_size > INT32_MAX)
    return PA_ERR_UNSUPPORTED;
  const bool f8 = is_8bit(cache->dtype);
  if (static_cast<int64_t>(max_context_len) > static_cast<int64_t>(max_blocks_per_seq) * cache->block_size ||
      max_q_len > max_context_len)
    return PA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  if (num_seqs == 0 || max_q_len == 0) return PA_OK;
  if (!q || !cu_q_lens || !block_tables || !context_lens || !out || !aligned16(q) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(cu_q_lens) & 3) || (reinterpret_cast<uintptr_t>(block_tables) & 3) ||
      (reinterpret_cast<uintptr_t>(context_lens) & 3))
    return PA_ERR_INVALID_ARG;
  // 128-row query tiles; at head_dim 128 two tiles of a sequence share one CTA
  const int tiles_per_cta = cache->head_dim == 128 ? 2 : 1;
  const int tt = 128 / G;
  const int64_t ntiles = ((static_cast<int64_t>(max_q_len) + tt - 1) / tt + tiles_per_cta - 1) / tiles_per_cta;
  if (num_seqs > 65535 || ntiles > 65535) return PA_ERR_UNSUPPORTED;
  PrefillArgs a;
  a.q = q;
  a.cu_q = cu_q_lens;
  a.tables = block_tables;
  a.lens = context_lens;
  a.out = out;
  a.num_blocks = cache->num_blocks;
  a.num_seqs = num_seqs;
  a.hq = num_q_heads;
  a.hkv = cache->num_kv_heads;
  a.bs = cache->block_size;
  a.max_blocks = max_blocks_per_seq;
  a.max_ctx = max_context_len;
  a.ntiles = static_cast<int32_t>(ntiles);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.v_scale = 1.f;
  if (f8) {
    // q . (k_scale * code) = (k_scale * q) . code; the V scale multiplies O.
    a.scale_log2 *= cache->k_scale;
    a.v_scale = cache->v_scale;
  }
  a.group_offs = a.group_members = a.group_prefix = nullptr;
  a.prefix_part_tokens = a.max_parts = a.parts_stride = 0;
  a.ws_ml = a.ws_o = nullptr;
  CUtensorMap tk, tv, to, tq;
  const uint64_t rows = static_cast<uint64_t>(cache->num_blocks) * cache->num_kv_heads * cache->block_size;
  auto enc = f8 ? encode_rows_u8 : encode_rows;
  if (!enc(&tk, cache->k, rows, cache->head_dim, cache->block_size) ||
      !enc(&tv, cache->v, rows, cache->head_dim, cache->block_size) ||
      !encode_out_tiles(&to, out, static_cast<uint64_t>(num_seqs) * max_q_len, num_q_heads, cache->head_dim, G) ||
      !encode_q_tiles(&tq, const_cast<void*>(q), static_cast<uint64_t>(num_seqs) * max_q_len, num_q_heads,
                      cache->head_dim, G))
    return PA_ERR_CUDA;
  const dim3 grid(cache->num_kv_heads, num_seqs, static_cast<unsigned>(ntiles));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto launch = [&](auto kern, int threads, int smem) -> pa_status {
    if (!smem_attrs(reinterpret_cast<const void*>(kern), smem, false)) return PA_ERR_CUDA;
    kern<<<grid, threads, smem, s>>>(tk, tv, to, tq, a);
    return launched();
  };
  auto launch8 = [&](auto cf) -> pa_status {
    constexpr int CF = decltype(cf)::value;
    using F128 = TcCfg<128, 2, true>;
    using F64 = TcCfg<64, 1, true>;
    if (cache->head_dim == 128) {
      switch (G) {
        case 1: return launch(prefill_tc_kernel<128, 1, 2, CF>, F128::kThreads, F128::kSmemBytes);
        case 2: return launch(prefill_tc_kernel<128, 2, 2, CF>, F128::kThreads, F128::kSmemBytes);
        case 4: return launch(prefill_tc_kernel<128, 4, 2, CF>, F128::kThreads, F128::kSmemBytes);
        default: return launch(prefill_tc_kernel<128, 8, 2, CF>, F128::kThreads, F128::kSmemBytes);
      }
    }
    switch (G) {
      case 1: return launch(prefill_tc_kernel<64, 1, 1, CF>, F64::kThreads, F64::kSmemBytes);
      case 2: return launch(prefill_tc_kernel<64, 2, 1, CF>, F64::kThreads, F64::kSmemBytes);
      case 4: return launch(prefill_tc_kernel<64, 4, 1, CF>, F64::kThreads, F64::kSmemBytes);
      default: return launch(prefill_tc_kernel<64, 8, 1, CF>, F64::kThreads, F64::kSmemBytes);
    }
  };
  if (f8)
    return cache->dtype == PA_INT8 ? launch8(std::integral_constant<int, kCodeS8>{})
                                   : launch8(std::integral_constant<int, kCodeE4M3>{});
  using C128 = TcCfg<128, 2>;
  using C64 = TcCfg<64, 1>;
  if (cache->head_dim == 128) {
    switch (G) {
      case 1: return launch(prefill_tc_kernel<128, 1, 2>, C128::kThreads, C128::kSmemBytes);
      case 2: return launch(prefill_tc_kernel<128, 2, 2>, C128::kThreads, C128::kSmemBytes);
      case 4: return launch(prefill_tc_kernel<128, 4, 2>, C128::kThreads, C128::kSmemBytes);
      default: return launch(prefill_tc_kernel<128, 8, 2>, C128::kThreads, C128::kSmemBytes);
    }
  }
  switch (G) {
    case 1: return launch(prefill_tc_kernel<64, 1, 1>, C64::kThreads, C64::kSmemBytes);
    case 2: return launch(prefill_tc_kernel<64, 2, 1>, C64::kThreads, C64::kSmemBytes);
    case 4: return launch(prefill_tc_kernel<64, 4, 1>, C64::kThreads, C64::kSmemBytes);
    default: return launch(prefill_tc_kernel<64, 8, 1>, C64::kThreads, C64::kSmemBytes);
  }
}

// Shared-prefix decode: prefix partitions of this many tokens (a multiple of
// the 64-token chunk).
#ifndef PA_CASCADE_PREFIX_PART
#define PA_CASCADE_PREFIX_PART 256
#endif
constexpr int32_t kCascadePrefixPart = PA_CASCADE_PREFIX_PART;

size_t cascade_ws_bytes(int32_t num_seqs, int32_t hq, int32_t hkv, int32_t D, int32_t suffix_parts,
                        int32_t prefix_parts) {
  const int32_t stride = suffix_parts + prefix_parts;
  return counters_bytes(num_seqs, hkv) + ml_bytes(num_seqs, hq, stride) +
         static_cast<size_t>(num_seqs) * hq * stride * D * 4;
}

size_t pa_decode_cascade_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                         int32_t max_context_len, int32_t block_size, int32_t max_prefix_tokens) {
  if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      max_prefix_tokens < 0)
    return 0;
  const int32_t P = resolve_partition(num_seqs, num_kv_heads, max_context_len, block_size, -1);
  return cascade_ws_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, num_parts(max_context_len, P),
                          (max_prefix_tokens + kCascadePrefixPart - 1) / kCascadePrefixPart);
}

pa_status pa_decode_cascade(const void* q, int32_t num_seqs, int32_t num_q_heads, const pa_cache* cache,
                            const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                            int32_t max_context_len, int32_t num_groups, const int32_t* group_offsets,
                            const int32_t* group_members, const int32_t* group_prefix_tokens,
                            const int32_t* seq_prefix_tokens, int32_t max_group_size, int32_t max_prefix_tokens,
                            const int32_t* seq_order, float scale, float* out, void* workspace,
                            size_t workspace_bytes, pa_stream stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || num_q_heads <= 0 || max_blocks_per_seq <= 0 || max_context_len < 0 || num_groups < 0 ||
      max_group_size < 0 || max_prefix_tokens < 0 || max_prefix_tokens > max_context_len)
    return PA_ERR_INVALID_ARG;
  if (num_q_heads % cache->num_kv_heads) return PA_ERR_INVALID_ARG;
  const int G = num_q_heads / cache->num_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
  if ((cache->dtype != PA_BF16 && !is_8bit(cache->dtype)) || cache->block_size < 8) return PA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(cache->num_blocks) * cache->num_kv_heads * cache->block_size > INT32_MAX)
    return PA_ERR_UNSUPPORTED;
  if (max_group_size > 64 / G) return PA_ERR_INVALID_ARG;  // one 64-row tile per group
  if (static_cast<int64_t>(max_context_len) > static_cast<int64_t>(max_blocks_per_seq) * cache->block_size)
    return PA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  if (num_seqs == 0) return PA_OK;
  if (!q || !block_tables || !context_lens || !out || !seq_prefix_tokens || !aligned16(q) || !aligned16(out) ||
      (num_groups > 0 && (!group_offsets || !group_members || !group_prefix_tokens)) ||
      (reinterpret_cast<uintptr_t>(seq_order) & 3))
    return PA_ERR_INVALID_ARG;
  if (num_seqs > 65535 || num_groups > 65535) return PA_ERR_UNSUPPORTED;

  const int32_t P = resolve_partition(num_seqs, cache->num_kv_heads, max_context_len, cache->block_size, -1);
  const int32_t parts = num_parts(max_context_len, P);
  const int32_t pparts = (max_prefix_tokens + kCascadePrefixPart - 1) / kCascadePrefixPart;
  const size_t need = cascade_ws_bytes(num_seqs, num_q_heads, cache->num_kv_heads, cache->head_dim, parts, pparts);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255)) return PA_ERR_INVALID_ARG;
  char* ws = static_cast<char*>(workspace);
  const int32_t stride = parts + pparts;
  const size_t cb = counters_bytes(num_seqs, cache->num_kv_heads);
  float* ws_ml = reinterpret_cast<float*>(ws + cb);
  float* ws_o = reinterpret_cast<float*>(ws + cb + ml_bytes(num_seqs, num_q_heads, stride));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int D = cache->head_dim;

  // 1. prefix partials: one CTA per (kv head, prefix partition, group), rows = members x heads
  if (num_groups > 0 && pparts > 0) {
    PrefillArgs pa;
    pa.q = q;
    pa.cu_q = nullptr;
    pa.tables = block_tables;
    pa.lens = context_lens;
    pa.out = nullptr;
    pa.num_blocks = cache->num_blocks;
    pa.num_seqs = num_seqs;
    pa.hq = num_q_heads;
    pa.hkv = cache->num_kv_heads;
    pa.bs = cache->block_size;
    pa.max_blocks = max_blocks_per_seq;
    pa.max_ctx = max_context_len;
    pa.ntiles = 0;
    pa.scale_log2 = scale * 1.4426950408889634f;
    pa.v_scale = 1.f;
    if (is_8bit(cache->dtype)) {
      // q . (k_scale * code) = (k_scale * q) . code; the V scale multiplies the partial o.
      pa.scale_log2 *= cache->k_scale;
      pa.v_scale = cache->v_scale;
    }
    pa.group_offs = group_offsets;
    pa.group_members = group_members;
    pa.group_prefix = group_prefix_tokens;
    pa.prefix_part_tokens = kCascadePrefixPart;
    pa.max_parts = parts;
    pa.parts_stride = stride;
    pa.ws_ml = ws_ml;
    pa.ws_o = ws_o;
    CUtensorMap tk, tv;
    const uint64_t rows = static_cast<uint64_t>(cache->num_blocks) * cache->num_kv_heads * cache->block_size;
    bool enc_ok;
    if (is_8bit(cache->dtype))
      enc_ok = encode_rows_u8(&tk, cache->k, rows, D, cache->block_size) &&
               encode_rows_u8(&tv, cache->v, rows, D, cache->block_size);
    else if (D == 128)  // one copy per (block, head) tile, as the grouped-head decode
      enc_ok = encode_rows_halves(&tk, cache->k, rows, cache->block_size) &&
               encode_rows_halves(&tv, cache->v, rows, cache->block_size);
    else
      enc_ok = encode_rows(&tk, cache->k, rows, D, cache->block_size) &&
               encode_rows(&tv, cache->v, rows, D, cache->block_size);
    if (!enc_ok) return PA_ERR_CUDA;
    const dim3 grid(cache->num_kv_heads, pparts, num_groups);
    auto launch = [&](auto kern, int smem) -> pa_status {
      // the largest shared-memory carveout: two of these CTAs fit an SM
      if (!smem_attrs(reinterpret_cast<const void*>(kern), smem, true)) return PA_ERR_CUDA;
      kern<<<grid, MmaCfg<128>::kThreads, smem, s>>>(tk, tv, pa);
      return launched();
    };
    auto launch_cf = [&](auto cf) -> pa_status {
      constexpr int CF = decltype(cf)::value;
      constexpr int S128 = prefill_mma_smem_bytes<128, CF>(), S64 = prefill_mma_smem_bytes<64, CF>();
      if (D == 128)
        return G == 1 ? launch(prefill_mma_kernel<128, 1, true, CF>, S128)
             : G == 2 ? launch(prefill_mma_kernel<128, 2, true, CF>, S128)
             : G == 4 ? launch(prefill_mma_kernel<128, 4, true, CF>, S128)
                      : launch(prefill_mma_kernel<128, 8, true, CF>, S128);
      return G == 1 ? launch(prefill_mma_kernel<64, 1, true, CF>, S64)
           : G == 2 ? launch(prefill_mma_kernel<64, 2, true, CF>, S64)
           : G == 4 ? launch(prefill_mma_kernel<64, 4, true, CF>, S64)
                    : launch(prefill_mma_kernel<64, 8, true, CF>, S64);
    };
    st = cache->dtype == PA_INT8       ? launch_cf(std::integral_constant<int, kCodeS8>{})
         : cache->dtype == PA_FP8_E4M3 ? launch_cf(std::integral_constant<int, kCodeE4M3>{})
                                       : launch_cf(std::integral_constant<int, 0>{});
    if (st != PA_OK) return st;
  }

  // 2. suffix partials: the decode kernels over [seq_prefix_tokens[s], L_s)
  DecodeArgs a;
  a.q = q;
  a.kc = cache->k;
  a.vc = cache->v;
  a.tables = block_tables;
  a.lens = context_lens;
  a.out = out;
  a.counters = reinterpret_cast<unsigned int*>(ws);
  a.ws_ml = ws_ml;
  a.ws_o = ws_o;
  a.num_blocks = cache->num_blocks;
  a.num_seqs = num_seqs;
  a.hq = num_q_heads;
  a.hkv = cache->num_kv_heads;
  a.bs = cache->block_size;
  a.max_blocks = max_blocks_per_seq;
  a.max_ctx = max_context_len;
  a.part_tokens = parts > 1 ? P : 0;
  a.max_parts = parts;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.n_items = static_cast<int32_t>(static_cast<int64_t>(cache->num_kv_heads) * num_seqs * parts);
  a.starts = seq_prefix_tokens;
  a.force_partials = 1;
  a.parts_stride = stride;
  a.prefix_part_tokens = kCascadePrefixPart;
  // unsplit suffixes: each suffix CTA merges its sequence's prefix partials itself
  a.cascade_direct = parts == 1 ? 1 : 0;
  a.seq_order = seq_order;
  // the suffix pass runs alongside the prefix pass (launched just before it on
  // this stream) and waits for it only where it folds in the prefix partials
  a.after_prefix_pass = a.cascade_direct && num_groups > 0 && pparts > 0 ? 1 : 0;
  if (is_8bit(cache->dtype)) {
    a.scale_log2 *= cache->k_scale;
    a.v_scale = cache->v_scale;
  }
  const dim3 grid(cache->num_kv_heads, num_seqs, parts);
  if (mma_eligible(cache, G)) {
    st = dispatch_mma(a, cache, G, s);
  } else if (f8_mma_eligible(cache)) {
    st = D == 128 ? dispatch_f8<128>(a, cache, G, grid, s) : dispatch_f8<64>(a, cache, G, grid, s);
  } else if (cache->dtype == PA_BF16) {
    st = D == 128 ? dispatch_g<__nv_bfloat16, 128>(a, G, grid, s) : dispatch_g<__nv_bfloat16, 64>(a, G, grid, s);
  } else {
    return PA_ERR_UNSUPPORTED;  // unreachable: an 8-bit cache here has block_size >= 8
  }
  if (st != PA_OK || a.cascade_direct) return st;
  // 3. merge prefix and suffix partials (split suffixes)
  return D == 128 ? launch_reduce<128>(a, s) : launch_reduce<64>(a, s);
}

int32_t pa_decode_partition_tokens(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                   int32_t max_context_len, int32_t block_size) {
  (void)num_q_heads;
  return resolve_partition(num_seqs, num_kv_heads, max_context_len, block_size, -1);
}

int32_t pa_decode_ordered_partition_tokens(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                           int32_t max_context_len, int32_t block_size) {
  (void)num_q_heads;
  return resolve_partition(num_seqs, num_kv_heads, max_context_len, block_size, -1, true);
}

size_t pa_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                 int32_t max_context_len, int32_t block_size, int32_t partition_tokens) {
  if (num_seqs <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0) return 0;
  const int32_t P = resolve_partition(num_seqs, num_kv_heads, max_context_len, block_size, partition_tokens);
  return ws_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, num_parts(max_context_len, P));
}

namespace {

// k_new / v_new / slot_mapping non-null: the fused KV append of pa_decode_append.
pa_status decode_impl(const void* q, int32_t num_seqs, int32_t num_q_heads, const pa_cache* cache,
                      const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                      int32_t max_context_len, const int32_t* seq_order, float scale, float* out,
                      int32_t partition_tokens, void* workspace, size_t workspace_bytes, pa_stream stream,
                      const void* k_new = nullptr, const void* v_new = nullptr,
                      const int64_t* slot_mapping = nullptr) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || num_q_heads <= 0 || max_blocks_per_seq <= 0 || max_context_len < 0) return PA_ERR_INVALID_ARG;
  if (num_q_heads % cache->num_kv_heads) return PA_ERR_INVALID_ARG;
  const int G = num_q_heads / cache->num_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(max_context_len) > static_cast<int64_t>(max_blocks_per_seq) * cache->block_size)
    return PA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  if (partition_tokens < -1 || (partition_tokens > 0 && partition_tokens % cache->block_size))
    return PA_ERR_INVALID_ARG;
  if (num_seqs == 0) return PA_OK;
  if (!q || !block_tables || !context_lens || !out || !aligned16(q) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(block_tables) & 3) || (reinterpret_cast<uintptr_t>(context_lens) & 3) ||
      (reinterpret_cast<uintptr_t>(seq_order) & 3))
    return PA_ERR_INVALID_ARG;
  if (slot_mapping && (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new) ||
                       (reinterpret_cast<uintptr_t>(slot_mapping) & 7)))
    return PA_ERR_INVALID_ARG;
  if (num_seqs > 65535) return PA_ERR_UNSUPPORTED;

  const int32_t P = resolve_partition(num_seqs, cache->num_kv_heads, max_context_len, cache->block_size,
                                      partition_tokens, seq_order != nullptr);
  const int32_t parts = num_parts(max_context_len, P);
  if (parts > 65535 || static_cast<int64_t>(cache->num_kv_heads) * num_seqs * parts > INT32_MAX)
    return PA_ERR_UNSUPPORTED;
  const size_t need = ws_bytes(num_seqs, num_q_heads, cache->num_kv_heads, cache->head_dim, parts);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255)) return PA_ERR_INVALID_ARG;

  DecodeArgs a;
  a.q = q;
  a.kc = cache->k;
  a.vc = cache->v;
  a.tables = block_tables;
  a.lens = context_lens;
  a.out = out;
  char* ws = static_cast<char*>(workspace);
  a.counters = reinterpret_cast<unsigned int*>(ws);
  const size_t cb = counters_bytes(num_seqs, cache->num_kv_heads);
  a.ws_ml = parts > 1 ? reinterpret_cast<float*>(ws + cb) : nullptr;
  a.ws_o = parts > 1 ? reinterpret_cast<float*>(ws + cb + ml_bytes(num_seqs, num_q_heads, parts)) : nullptr;
  a.num_blocks = cache->num_blocks;
  a.num_seqs = num_seqs;
  a.hq = num_q_heads;
  a.hkv = cache->num_kv_heads;
  a.bs = cache->block_size;
  a.max_blocks = max_blocks_per_seq;
  a.max_ctx = max_context_len;
  a.part_tokens = parts > 1 ? P : 0;
  a.max_parts = parts;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.n_items = static_cast<int32_t>(static_cast<int64_t>(cache->num_kv_heads) * num_seqs * parts);
  a.starts = nullptr;
  a.force_partials = 0;
  a.parts_stride = parts;
  a.prefix_part_tokens = 0;
  a.seq_order = seq_order;
  a.k_new = k_new;
  a.v_new = v_new;
  a.slot_mapping = slot_mapping;
  a.num_slots = static_cast<int64_t>(cache->num_blocks) * cache->block_size;
  a.k_scale_store = cache->k_scale;
  a.v_scale_store = cache->v_scale;
  if (is_8bit(cache->dtype)) {
    // q . (k_scale * code) = (k_scale * q) . code; the V scale multiplies o.
    a.scale_log2 *= cache->k_scale;
    a.v_scale = cache->v_scale;
    if (!std::isfinite(a.scale_log2)) return PA_ERR_INVALID_ARG;
  }

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  dim3 grid(cache->num_kv_heads, num_seqs, parts);
  const int D = cache->head_dim;
  // With few partitions per sequence the CTA that finishes a (sequence, kv
  // head) last merges its partials (no merge launch); many partitions keep the
  // merge kernel, which spreads the rows over the whole GPU.
  if (parts > 1 && parts < kFuseMergeMaxParts) {
    a.fuse_merge = 1;
    // (the persistent kernel's launch clears the counters itself)
    if (!(mma_eligible(cache, G) && mma_persistent(a)) &&
        cudaMemsetAsync(a.counters, 0, counters_bytes(num_seqs, cache->num_kv_heads), s) != cudaSuccess)
      return PA_ERR_CUDA;
  }
  if (mma_eligible(cache, G)) {
    st = dispatch_mma(a, cache, G, s);
  } else if (f8_mma_eligible(cache)) {
    st = D == 128 ? dispatch_f8<128>(a, cache, G, grid, s) : dispatch_f8<64>(a, cache, G, grid, s);
  } else if (cache->dtype == PA_FP8_E4M3) {
    st = D == 128 ? dispatch_g<__nv_fp8_e4m3, 128>(a, G, grid, s) : dispatch_g<__nv_fp8_e4m3, 64>(a, G, grid, s);
  } else if (cache->dtype == PA_INT8) {
    st = D == 128 ? dispatch_g<int8_t, 128>(a, G, grid, s) : dispatch_g<int8_t, 64>(a, G, grid, s);
  } else if (cache->dtype == PA_BF16) {
    st = D == 128 ? dispatch_g<__nv_bfloat16, 128>(a, G, grid, s) : dispatch_g<__nv_bfloat16, 64>(a, G, grid, s);
  } else {
    st = D == 128 ? dispatch_g<float, 128>(a, G, grid, s) : dispatch_g<float, 64>(a, G, grid, s);
  }
  if (st != PA_OK || parts <= 1 || a.fuse_merge) return st;
  return D == 128 ? launch_reduce<128>(a, s) : launch_reduce<64>(a, s);
}

}  // namespace

pa_status pa_decode(const void* q, int32_t num_seqs, int32_t num_q_heads, const pa_cache* cache,
                    const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                    int32_t max_context_len, float scale, float* out, int32_t partition_tokens, void* workspace,
                    size_t workspace_bytes, pa_stream stream) {
  return decode_impl(q, num_seqs, num_q_heads, cache, block_tables, max_blocks_per_seq, context_lens,
                     max_context_len, nullptr, scale, out, partition_tokens, workspace, workspace_bytes, stream);
}

pa_status pa_decode_ordered(const void* q, int32_t num_seqs, int32_t num_q_heads, const pa_cache* cache,
                            const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                            int32_t max_context_len, const int32_t* seq_order, float scale, float* out,
                            int32_t partition_tokens, void* workspace, size_t workspace_bytes, pa_stream stream) {
  return decode_impl(q, num_seqs, num_q_heads, cache, block_tables, max_blocks_per_seq, context_lens,
                     max_context_len, seq_order, scale, out, partition_tokens, workspace, workspace_bytes, stream);
}

pa_status pa_decode_append(const void* q, const void* k_new, const void* v_new, const int64_t* slot_mapping,
                           int32_t num_seqs, int32_t num_q_heads, const pa_cache* cache, const int32_t* block_tables,
                           int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t max_context_len,
                           const int32_t* seq_order, float scale, float* out, int32_t partition_tokens,
                           void* workspace, size_t workspace_bytes, pa_stream stream) {
  if (!slot_mapping) return PA_ERR_INVALID_ARG;
  return decode_impl(q, num_seqs, num_q_heads, cache, block_tables, max_blocks_per_seq, context_lens,
                     max_context_len, seq_order, scale, out, partition_tokens, workspace, workspace_bytes, stream,
                     k_new, v_new, slot_mapping);
}

pa_status pa_selftest_wait_timeout(int64_t timeout_ns, pa_stream stream) {
  if (timeout_ns <= 0 || timeout_ns > 10000000000ll) return PA_ERR_INVALID_ARG;
  selftest_wait_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint64_t>(timeout_ns));
  return launched();
}

pa_status pa_get_device_error(pa_stream stream, int64_t* info_out) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PA_ERR_CUDA;
  unsigned long long w = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&w, pa::g_error_word, sizeof(w)) != cudaSuccess) return PA_ERR_CUDA;
  if (w == 0) {
    if (info_out) *info_out = 0;
    return PA_OK;
  }
  if (cudaMemcpyToSymbol(pa::g_error_word, &zero, sizeof(zero)) != cudaSuccess) return PA_ERR_CUDA;
  if (info_out) *info_out = static_cast<int64_t>(static_cast<int32_t>(w & 0xffffffffull));
  return static_cast<pa_status>(w >> 32);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free decode (pa_decode_static_workspace).
//
// For callers that are handed only inputs and outputs and may not allocate
// device memory (a runtime that owns the whole device, or a serving loop where
// cudaMalloc's possible device synchronisation is not allowed), the split
// partials live in this fixed array instead of a caller workspace. Every
// device that loads the library holds it until the process exits.
namespace {

static __device__ __align__(256) unsigned char g_static_ws[PA_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;

// In host code g_static_ws names a host-side stand-in, not device memory, so
// the device address is looked up once per device (with that device current)
// and cached. The first call on a device therefore makes a runtime query.
void* static_ws_address(pa_status* st) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *st = PA_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || !p) {
      *st = PA_ERR_CUDA;
      return nullptr;
    }
    addr[dev] = p;
  }
  *st = PA_OK;
  return addr[dev];
}

}  // namespace

extern "C" pa_status pa_decode_static_workspace(const void* q, int32_t num_seqs, int32_t num_q_heads,
                                                const pa_cache* cache, const int32_t* block_tables,
                                                int32_t max_blocks_per_seq, const int32_t* context_lens,
                                                int32_t max_context_len, float scale, float* out,
                                                int32_t partition_tokens, pa_stream stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || num_q_heads <= 0 || partition_tokens < -1) return PA_ERR_INVALID_ARG;
  const size_t need = pa_decode_workspace_bytes(num_seqs, num_q_heads, cache->num_kv_heads, cache->head_dim,
                                                max_context_len, cache->block_size, partition_tokens);
  if (need > PA_STATIC_WORKSPACE_BYTES) return PA_ERR_INVALID_ARG;
  void* ws = nullptr;
  if (need > 0) {
    ws = static_ws_address(&st);
    if (st != PA_OK) return st;
  }
  return pa_decode(q, num_seqs, num_q_heads, cache, block_tables, max_blocks_per_seq, context_lens, max_context_len,
                   scale, out, partition_tokens, ws, need > 0 ? PA_STATIC_WORKSPACE_BYTES : 0, stream);
}
