// attn.cu -- the attention prologue of a layer: fused Q/K RMS normalisation,
// rotary embedding and KV-cache write ("[Model] Add Flint (RecursiveSI/flint)",
// section "What happened": one fused kernel in the per-layer decode chain).
// Shapes from "Recursive Flint: 125 tok/s on an M4 Pro", architecture table:
// 32 query and 4 key/value heads of dimension 128; rotary positions on the
// sliding-window layers, none on the full-attention layers (rope = 0).
//
// One half-warp per (token, head) of the fused projection qkv
// [T][Hq + 2*Hkv][128] bf16: lane l of the half holds elements 8l..8l+7 (one
// 16-byte load; a half-warp reads a head's 256 contiguous bytes). Query/key
// heads: sum of squares by a 16-lane reduction, y = x / sqrt(mean + eps) * w
// in fp32; rotation partner of element i is i +- 64, held by lane l ^ 8 in
// the same register, so one shuffle per element; the cos/sin row of the
// token's position is read as four 16-byte loads per lane. Query heads go to q_out [T][Hq][128]; key heads to
// k_cache[slot][Hkv][128]; value heads are copied to v_cache[slot][Hkv][128].
// HBM-bound: 21,000 bytes per token at Hq = 32, Hkv = 4 (read qkv 10,240, the
// cos/sin row 512, position and slot 8; write q 8,192, k and v 1,024 each).
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "flint_moe.h"
#include "common.cuh"

namespace flint {
namespace {

constexpr int kHeadDim = 128;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

struct AttnPrologueParams {
  const uint16_t* qkv;
  const uint16_t* q_w;
  const uint16_t* k_w;
  const float* cos_sin;  // [max_pos][128]: cos in columns 0..63, sin in 64..127
  const int32_t* positions;
  const int32_t* slots;
  uint16_t* q_out;
  uint16_t* k_cache;
  uint16_t* v_cache;
  int32_t* status;  // nullable: FLINT_DEVCHECK_INDEX for a position or slot outside its range
  int T, Hq, Hkv, max_pos, rope;
  long long n_slots;
  float eps;
};

__global__ void __launch_bounds__(256) k_qk_norm_rope_kv(AttnPrologueParams p) {
  // half-warp per (token, head): lane l of the half holds elements 8l .. 8l+7.
  // The two halves of a warp may take different branches (a value head returns
  // early beside a query or key head), so shuffles name only this half's lanes.
  const int lane = threadIdx.x & 15;
  const unsigned hmask = 0xFFFFu << (threadIdx.x & 16);
  const int H = p.Hq + 2 * p.Hkv;
  const int task = blockIdx.x * 16 + (threadIdx.x >> 4);
  if (task >= p.T * H) return;
  const int t = task / H, h = task - t * H;
  const uint4 raw = __ldg(reinterpret_cast<const uint4*>(p.qkv + static_cast<size_t>(task) * kHeadDim) + lane);
  long long slot = -1;
  if (h >= p.Hq) {
    slot = p.slots[t];
    if (slot < 0 || slot >= p.n_slots) {
      if (lane == 0 && p.status != nullptr) atomicOr(p.status, FLINT_DEVCHECK_INDEX);
      return;
    }
  }
  if (h >= p.Hq + p.Hkv) {  // value head: copied to its cache slot
    uint16_t* dst = p.v_cache + (slot * p.Hkv + (h - p.Hq - p.Hkv)) * kHeadDim;
    reinterpret_cast<uint4*>(dst)[lane] = raw;
    return;
  }
  const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
  float x[8];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    x[2 * q] = bf16_lo(rw[q]);
    x[2 * q + 1] = bf16_hi(rw[q]);
  }
  const uint16_t* wv = h < p.Hq ? p.q_w : p.k_w;
  const uint4 wr = __ldg(reinterpret_cast<const uint4*>(wv) + lane);
  const uint32_t ww[4] = {wr.x, wr.y, wr.z, wr.w};
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) ss = fmaf(x[j], x[j], ss);
  // sum over the 16 lanes of this half-warp (xor offsets below 16 stay in it)
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(hmask, ss, o);
  const float r = 1.f / sqrtf(ss / static_cast<float>(kHeadDim) + p.eps);
  float y[8];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    y[2 * q] = x[2 * q] * r * bf16_lo(ww[q]);
    y[2 * q + 1] = x[2 * q + 1] * r * bf16_hi(ww[q]);
  }
  if (p.rope) {
    const int pos = p.positions[t];
    const bool bad = pos < 0 || pos >= p.max_pos;
    if (bad && lane == 0 && p.status != nullptr) atomicOr(p.status, FLINT_DEVCHECK_INDEX);
    // pair index c = element mod 64: lanes 0..7 of a half hold the first
    // halves, lanes 8..15 the second halves of the same pairs
    const int c = 8 * (lane & 7);
    float cc[8], sn[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      cc[j] = 1.f;
      sn[j] = 0.f;
    }
    if (!bad) {
      const float* row = p.cos_sin + static_cast<size_t>(pos) * kHeadDim;
      const float4 c0 = __ldg(reinterpret_cast<const float4*>(row + c));
      const float4 c1 = __ldg(reinterpret_cast<const float4*>(row + c + 4));
      const float4 s0 = __ldg(reinterpret_cast<const float4*>(row + 64 + c));
      const float4 s1 = __ldg(reinterpret_cast<const float4*>(row + 64 + c + 4));
      cc[0] = c0.x; cc[1] = c0.y; cc[2] = c0.z; cc[3] = c0.w;
      cc[4] = c1.x; cc[5] = c1.y; cc[6] = c1.z; cc[7] = c1.w;
      sn[0] = s0.x; sn[1] = s0.y; sn[2] = s0.z; sn[3] = s0.w;
      sn[4] = s1.x; sn[5] = s1.y; sn[6] = s1.z; sn[7] = s1.w;
    }
    const bool first = lane < 8;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float partner = __shfl_xor_sync(hmask, y[j], 8);
      // first half: y cos - partner sin; second half: y cos + partner sin
      y[j] = first ? fmaf(y[j], cc[j], -partner * sn[j]) : fmaf(y[j], cc[j], partner * sn[j]);
    }
  }
  const uint4 o = make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                             pack_bf16x2(y[6], y[7]));
  uint16_t* dst = h < p.Hq ? p.q_out + (static_cast<size_t>(t) * p.Hq + h) * kHeadDim
                           : p.k_cache + (slot * p.Hkv + (h - p.Hq)) * kHeadDim;
  reinterpret_cast<uint4*>(dst)[lane] = o;
}

bool aligned16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }


}  // namespace
}  // namespace flint

using namespace flint;

extern "C" int flint_qk_norm_rope_kv(const uint16_t* qkv, int32_t T, int32_t n_q_heads, int32_t n_kv_heads,
                                     int32_t head_dim, const uint16_t* q_norm_w, const uint16_t* k_norm_w,
                                     const float* cos_sin, int32_t max_pos, const int32_t* positions,
                                     int32_t rope, float eps, const int32_t* slots, int64_t n_slots,
                                     uint16_t* q_out, uint16_t* k_cache, uint16_t* v_cache, int32_t* status,
                                     void* stream) {
  if (head_dim != kHeadDim) return flint_fail_external(FLINT_ERR_UNSUPPORTED_SHAPE, "head_dim must be 128");
  if (T < 0 || n_q_heads < 1 || n_kv_heads < 1 || n_slots < 0 || !(eps >= 0.f))
    return flint_fail_external(FLINT_ERR_INVALID_ARG, "flint_qk_norm_rope_kv: bad sizes");
  if (T == 0) return FLINT_OK;
  if (!qkv || !q_norm_w || !k_norm_w || !slots || !q_out || !k_cache || !v_cache ||
      (rope && (!cos_sin || !positions || max_pos < 1)))
    return flint_fail_external(FLINT_ERR_INVALID_ARG, "flint_qk_norm_rope_kv: NULL pointer");
  if (!aligned16(qkv) || !aligned16(q_norm_w) || !aligned16(k_norm_w) || !aligned16(q_out) || !aligned16(k_cache) ||
      !aligned16(v_cache) || (rope && !aligned16(cos_sin)))
    return flint_fail_external(FLINT_ERR_MISALIGNED, "flint_qk_norm_rope_kv: misaligned pointer");
  AttnPrologueParams p{};
  p.qkv = qkv;
  p.q_w = q_norm_w;
  p.k_w = k_norm_w;
  p.cos_sin = cos_sin;
  p.positions = positions;
  p.slots = slots;
  p.q_out = q_out;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.status = status;
  p.T = T;
  p.Hq = n_q_heads;
  p.Hkv = n_kv_heads;
  p.max_pos = max_pos;
  p.rope = rope ? 1 : 0;
  p.n_slots = n_slots;
  p.eps = eps;
  const long long tasks = static_cast<long long>(T) * (n_q_heads + 2 * n_kv_heads);
  if (tasks > 0x7fffffffLL) return flint_fail_external(FLINT_ERR_UNSUPPORTED_SHAPE, "too many tokens");
  const long long blocks = (tasks + 15) / 16;
  k_qk_norm_rope_kv<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return flint_fail_external(FLINT_ERR_CUDA, cudaGetErrorString(e));
  return FLINT_OK;
}
