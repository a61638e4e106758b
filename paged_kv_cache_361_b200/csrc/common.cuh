// Device helpers shared by the libpagedattn kernels: the per-device error
// word, mbarrier / bulk-copy (TMA) wrappers, and bf16 unpacking.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pagedattn.h"

namespace pa {

// First error recorded since the last pa_get_device_error: high 32 bits the
// pa_status, low 32 bits the offending value (truncated). Every kernel lives in
// the one translation unit capi.cu, which is the only includer of this header.
__device__ unsigned long long g_error_word = 0;

__device__ __forceinline__ void record_error(pa_status code, long long info) {
  unsigned long long w = (static_cast<unsigned long long>(code) << 32) | (static_cast<unsigned long long>(info) & 0xffffffffull);
  atomicCAS(&g_error_word, 0ull, w);
}

// Bounded waits: a kernel gives up an mbarrier wait after this much wall time
// (read from the %globaltimer nanosecond clock), far beyond any legitimate
// copy latency, records PA_ERR_DEVICE_TIMEOUT and returns.
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for phase `parity` of `bar`. Returns false (and records
// PA_ERR_DEVICE_TIMEOUT) if the phase did not complete within timeout_ns.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns = kWaitTimeoutNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t start = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 0 && global_timer_ns() - start > timeout_ns) {
      record_error(PA_ERR_DEVICE_TIMEOUT, 0);
      return false;
    }
  }
}

__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ uint64_t l2_evict_normal_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// L2 priority of the decode kernels' K/V reads. Every byte of a plain decode
// is read once per step, so evict-first keeps the stream from displacing
// other data; a block shared by several sequences of the batch (forked
// samples, cached prefixes) is read once per holder, and an evict-normal
// stream lets the later readers hit in L2.
#ifndef PA_KV_STREAM_POLICY
#define PA_KV_STREAM_POLICY 0
#endif
__device__ __forceinline__ uint64_t kv_stream_policy() {
#if PA_KV_STREAM_POLICY == 1
  return l2_evict_normal_policy();
#elif PA_KV_STREAM_POLICY == 2
  return l2_evict_last_policy();
#else
  return l2_evict_first_policy();
#endif
}

// One contiguous global -> shared copy by the TMA unit, completing on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Two e4m3 codes (low byte first) -> two floats (exact: every e4m3 value is
// representable in fp16 and fp32).
__device__ __forceinline__ float2 fp8x2_to_float2(uint16_t w) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w), __NV_E4M3);
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// x / scale in fp32 (IEEE division), rounded to the nearest e4m3 code (ties
// to even); finite values beyond +-448 and infinities saturate to +-448, NaN
// stays NaN.
__device__ __forceinline__ uint8_t quantize_e4m3(float x, float scale) {
  const float y = __fdiv_rn(x, scale);
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3));
}

// x / scale in fp32 (IEEE division), rounded to the nearest integer (ties to
// even) and clamped to [-127, 127] (infinities too); NaN becomes 0.
__device__ __forceinline__ int8_t quantize_s8(float x, float scale) {
  float y = __fdiv_rn(x, scale);
  y = y != y ? 0.f : fminf(fmaxf(y, -127.f), 127.f);
  return static_cast<int8_t>(__float2int_rn(y));
}

// Element formats of an 8-bit cache: e4m3 floats, or symmetric int8.
enum CodeFmt : int { kCodeE4M3 = 1, kCodeS8 = 2 };

// Four int8 codes (low byte first) -> four floats, exact: each byte, biased
// by 128, becomes the low byte of the fp32 2^23, whose unit is 1, and
// 2^23 + 128 is subtracted.
__device__ __forceinline__ void s8x4_to_float(uint32_t w, float (&f)[4]) {
  const uint32_t u = w ^ 0x80808080u;
  f[0] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540)) - 8388736.f;
  f[1] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7541)) - 8388736.f;
  f[2] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7542)) - 8388736.f;
  f[3] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7543)) - 8388736.f;
}

// 2^x by the hardware approximation (ex2.approx.ftz: relative error ~2^-22,
// results below 2^-126 flush to 0, 2^-inf = 0). Used for softmax weights.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Programmatic dependent launch (a grid launched with the
// programmatic-stream-serialization attribute may start before the previous
// grid on its stream has finished): the previous grid lets it start with
// launch_dependents; the dependent grid's wait returns once the previous grid
// has completed and its memory operations are visible. Both are no-ops when
// the grids were launched without the attribute.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Three-input maximum (one instruction on sm_100a; NaN-ignoring like fmaxf).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Packed fp32 pairs (one instruction for two lanes of arithmetic on sm_100a),
// each element rounded as the scalar operation would be.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 A, B, C, D;\n\tmov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\tmov.b64 C, {%6, %7};\n\t"
      "fma.rn.f32x2 D, A, B, C;\n\tmov.b64 {%0, %1}, D;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 A, B, D;\n\tmov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\t"
      "add.rn.f32x2 D, A, B;\n\tmov.b64 {%0, %1}, D;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// bf16 pair packed in a 32-bit word -> two floats (exact).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

}  // namespace pa
