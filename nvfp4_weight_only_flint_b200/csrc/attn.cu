// attn.cu -- the attention prologue of a layer: fused Q/K RMS normalisation,
// rotary embedding and KV-cache write ("[Model] Add Flint (RecursiveSI/flint)",
// section "What happened": one fused kernel in the per-layer decode chain).
// Shapes from "Recursive Flint: 125 tok/s on an M4 Pro", architecture table:
// 32 query and 4 key/value heads of dimension 128; rotary positions on the
// sliding-window layers, none on the full-attention layers (rope = 0).
//
// One warp per (token, head) of the fused projection qkv [T][Hq + 2*Hkv][128]
// bf16: lane l holds elements 4l..4l+3 (one 8-byte load; a warp reads a head's
// 256 contiguous bytes). Query/key heads: sum of squares by a warp reduction,
// y = x / sqrt(mean + eps) * w in fp32; rotation partner of element i is
// i +- 64, held by lane l ^ 16 in the same register, so one shuffle per
// element; the cos/sin row of the token's position is read as two 16-byte
// loads per lane. Query heads go to q_out [T][Hq][128]; key heads to
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
  const int lane = threadIdx.x & 31;
  const int H = p.Hq + 2 * p.Hkv;
  const long long task = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (task >= static_cast<long long>(p.T) * H) return;
  const int t = static_cast<int>(task / H), h = static_cast<int>(task % H);
  const uint2 raw = __ldg(reinterpret_cast<const uint2*>(p.qkv + task * kHeadDim) + lane);
  float x[4] = {bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y)};
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
    reinterpret_cast<uint2*>(dst)[lane] = raw;
    return;
  }
  const uint16_t* wv = h < p.Hq ? p.q_w : p.k_w;
  const uint2 wr = __ldg(reinterpret_cast<const uint2*>(wv) + lane);
  const float w[4] = {bf16_lo(wr.x), bf16_hi(wr.x), bf16_lo(wr.y), bf16_hi(wr.y)};
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) ss = fmaf(x[j], x[j], ss);
  ss = warp_sum(ss);
  const float r = 1.f / sqrtf(ss / static_cast<float>(kHeadDim) + p.eps);
  float y[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) y[j] = x[j] * r * w[j];
  if (p.rope) {
    const int pos = p.positions[t];
    const bool bad = pos < 0 || pos >= p.max_pos;
    if (bad && lane == 0 && p.status != nullptr) atomicOr(p.status, FLINT_DEVCHECK_INDEX);
    // pair index c = element mod 64: lanes 0..15 hold the first halves,
    // lanes 16..31 the second halves of the same pairs
    const int c = 4 * (lane & 15);
    float4 cs = make_float4(1.f, 1.f, 1.f, 1.f), sn = make_float4(0.f, 0.f, 0.f, 0.f);
    if (!bad) {
      const float* row = p.cos_sin + static_cast<size_t>(pos) * kHeadDim;
      cs = __ldg(reinterpret_cast<const float4*>(row + c));
      sn = __ldg(reinterpret_cast<const float4*>(row + 64 + c));
    }
    const float cc[4] = {cs.x, cs.y, cs.z, cs.w}, ssn[4] = {sn.x, sn.y, sn.z, sn.w};
    const bool first = lane < 16;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float partner = __shfl_xor_sync(0xffffffffu, y[j], 16);
      // first half: y cos - partner sin; second half: y cos + partner sin
      y[j] = first ? fmaf(y[j], cc[j], -partner * ssn[j]) : fmaf(y[j], cc[j], partner * ssn[j]);
    }
  }
  const uint2 o = make_uint2(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]));
  uint16_t* dst = h < p.Hq ? p.q_out + (static_cast<size_t>(t) * p.Hq + h) * kHeadDim
                           : p.k_cache + (slot * p.Hkv + (h - p.Hq)) * kHeadDim;
  reinterpret_cast<uint2*>(dst)[lane] = o;
}

bool aligned8(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 7u) == 0; }

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
  if (!aligned8(qkv) || !aligned8(q_norm_w) || !aligned8(k_norm_w) || !aligned8(q_out) || !aligned8(k_cache) ||
      !aligned8(v_cache) || (rope && (reinterpret_cast<uintptr_t>(cos_sin) & 15u)))
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
  const long long warps = static_cast<long long>(T) * (n_q_heads + 2 * n_kv_heads);
  const long long blocks = (warps + 7) / 8;
  if (blocks > 0x7fffffffLL) return flint_fail_external(FLINT_ERR_UNSUPPORTED_SHAPE, "too many tokens");
  k_qk_norm_rope_kv<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return flint_fail_external(FLINT_ERR_CUDA, cudaGetErrorString(e));
  return FLINT_OK;
}
