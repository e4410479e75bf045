// common.cuh -- sm_100a building blocks for the Flint MoE kernels: PTX wrappers
// (mbarrier, 1-D bulk copies, programmatic dependent launch), the in-register
// NVFP4 decode and the W4A16 dot product.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "flint_moe.h"

namespace flint {

// Records msg in the library's last-error slot (flint_last_error) and returns
// code; defined in flint_moe.cu.
int flint_fail_external(int code, const char* msg);

// Raises a kernel's dynamic shared-memory limit to the device's opt-in maximum,
// once per (kernel, current device); defined in flint_moe.cu.
cudaError_t flint_ensure_smem(const void* kern);

// A bounded device wait gives up after this many SM clock cycles (about one
// second at the B200's boost clock) and records FLINT_DEVCHECK_WAIT.
constexpr long long kWaitCycles = 2000000000LL;

// ----------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

// Make barrier initialisation visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity to complete. Returns false
// (and records FLINT_DEVCHECK_WAIT) if it did not complete in kWaitCycles.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) {
      atomicOr(status, FLINT_DEVCHECK_WAIT);
      return false;
    }
  }
  return true;
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`
// (16-byte aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Bring a span of global memory into L2 ahead of use (16-byte aligned, size a
// multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Tiled TMA loads through a tensor map (kernel-parameter or global address),
// completing on `bar`; x is the innermost coordinate (elements).
__device__ __forceinline__ void tma_load_2d(void* dst, const void* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const void* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
      : "memory");
}
// Programmatic dependent launch: wait for the preceding kernel's memory, and
// allow the following kernel to be scheduled.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint4 lds128(const void* p) {
  return *reinterpret_cast<const uint4*>(p);
}

// L2-coherent loads for data other CTAs of an earlier kernel wrote.
__device__ __forceinline__ float4 ldg_cg4(const float* p) {
  return __ldcg(reinterpret_cast<const float4*>(p));
}

// ----------------------------------------------------------------- NVFP4 decode
// Four E2M1 pairs (one 32-bit word = 8 codes, element 2i in the low nibble of
// byte i) -> four f16x2 registers holding the exact code values, element 2i in
// the low half.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t (&q)[4]) {
  asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %4;\n"
      " cvt.rn.f16x2.e2m1x2 %0, b0;\n cvt.rn.f16x2.e2m1x2 %1, b1;\n"
      " cvt.rn.f16x2.e2m1x2 %2, b2;\n cvt.rn.f16x2.e2m1x2 %3, b3;\n}"
      : "=r"(q[0]), "=r"(q[1]), "=r"(q[2]), "=r"(q[3])
      : "r"(w));
}

// Two E4M3 scale bytes (low byte first) -> their exact values as floats.
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint32_t two_bytes) {
  uint32_t h;
  const uint16_t b = static_cast<uint16_t>(two_bytes);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(b));
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// acc (f32) += q.lo * x.lo + q.hi * x.hi with f16 operands, products exact in
// f32 (sm_100 mixed-precision fma).
__device__ __forceinline__ void fma2_f16_f32(uint32_t q, uint32_t x, float& acc) {
  asm("{\n .reg .f16 ql, qh, xl, xh;\n mov.b32 {ql, qh}, %1;\n mov.b32 {xl, xh}, %2;\n"
      " fma.rn.f32.f16 %0, ql, xl, %0;\n fma.rn.f32.f16 %0, qh, xh, %0;\n}"
      : "+f"(acc)
      : "r"(q), "r"(x));
}

// acc (f32) += w.lo * x.lo + w.hi * x.hi with bf16 operands, products exact
// in f32, one rounding per step (sm_100 mixed-precision fma): the same result
// as fmaf on the widened values, without the widening instructions.
__device__ __forceinline__ void fma2_bf16_f32(uint32_t w, uint32_t x, float& acc) {
  asm("{\n .reg .b16 wl, wh, xl, xh;\n mov.b32 {wl, wh}, %1;\n mov.b32 {xl, xh}, %2;\n"
      " fma.rn.f32.bf16 %0, wl, xl, %0;\n fma.rn.f32.bf16 %0, wh, xh, %0;\n}"
      : "+f"(acc)
      : "r"(w), "r"(x));
}

// One 16-byte code vector (32 elements = two 16-element blocks) against TG
// activation vectors (16 f16x2 registers each, XS registers apart, pre-scaled
// by a power of two):
//   acc[t] += s_b0 * sum_{block 0} q*x + s_b1 * sum_{block 1} q*x.
template <int TG, int XS>
__device__ __forceinline__ void dot32_strided(const uint4 c, uint32_t scale2, const uint32_t* xh,
                                              float* acc) {
  uint32_t q[16];
  e2m1x8_to_f16x2(c.x, *reinterpret_cast<uint32_t(*)[4]>(&q[0]));
  e2m1x8_to_f16x2(c.y, *reinterpret_cast<uint32_t(*)[4]>(&q[4]));
  e2m1x8_to_f16x2(c.z, *reinterpret_cast<uint32_t(*)[4]>(&q[8]));
  e2m1x8_to_f16x2(c.w, *reinterpret_cast<uint32_t(*)[4]>(&q[12]));
  const float2 s = e4m3x2_to_f32x2(scale2);
#pragma unroll
  for (int t = 0; t < TG; ++t) {
    // two partial sums per block: dependency chains of 8 fused multiply-adds
    float p0a = 0.f, p0b = 0.f, p1a = 0.f, p1b = 0.f;
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      fma2_f16_f32(q[i], xh[t * XS + i], p0a);
      fma2_f16_f32(q[i + 1], xh[t * XS + i + 1], p0b);
      fma2_f16_f32(q[i + 8], xh[t * XS + i + 8], p1a);
      fma2_f16_f32(q[i + 9], xh[t * XS + i + 9], p1b);
    }
    acc[t] = fmaf(p0a + p0b, s.x, acc[t]);
    acc[t] = fmaf(p1a + p1b, s.y, acc[t]);
  }
}

// ----------------------------------------------------------------- activations
__device__ __forceinline__ float bf16_bits_to_f32(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}

// Power-of-two scale sigma with amax*sigma <= 2^15, so that every value of a
// row fits f16 without overflow (sigma = 1 when amax is 0).
__device__ __forceinline__ float pow2_scale_for(float amax) {
  if (!(amax > 0.f) || !isfinite(amax)) return 1.f;
  // amax = m * 2^e with m in [0.5, 1) (for subnormal amax e <= -126, and the
  // clamp below gives the same 2^127): e = biased exponent - 126
  const int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu) - 126;
  int p = 15 - e;
  p = max(-126, min(p, 127));
  return __uint_as_float(static_cast<uint32_t>(p + 127) << 23);
}

// Pack two floats (already scaled) into f16x2, element a in the low half.
__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ----------------------------------------------------------------- warp helpers
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sum over aligned segments of `seg` lanes (seg a power of two <= 32).
template <int SEG>
__device__ __forceinline__ float segment_sum(float v) {
#pragma unroll
  for (int o = SEG / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int SEG>
__device__ __forceinline__ float segment_max(float v) {
#pragma unroll
  for (int o = SEG / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// silu(g) * u, with silu(g) = g / (1 + e^-g).
__device__ __forceinline__ float swiglu(float g, float u) { return g / (1.f + expf(-g)) * u; }

}  // namespace flint
