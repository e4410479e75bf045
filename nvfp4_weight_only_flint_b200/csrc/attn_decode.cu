// attn_decode.cu -- grouped-query decode attention over the bf16 KV cache the
// attention prologue writes ("[Model] Add Flint (RecursiveSI/flint)", section
// "What happened": the per-layer decode chain; heads from "Recursive Flint:
// 125 tok/s on an M4 Pro", architecture table: 32 query and 4 key/value heads
// of dimension 128). Query token t, head h attends the cache rows start[t] ..
// start[t] + len[t] - 1 of key/value head g = h / group (group = Hq / Hkv):
// o = softmax(scale * q . k) v.
//
// Split-K "flash decoding" on the register-fragment tensor cores.
// k_attn_partial: one CTA per (context chunk, kv head g, token t). Its four
// warps split the chunk; each streams its keys in blocks of 16 through a
// three-stage cp.async ring of shared memory (16 key and 16 value rows of 256
// bytes, padded to 272 so ldmatrix rows hit distinct banks). The group's query
// heads are rows of one m16n8k16 tile (rows >= group zero):
//   S [head][16 keys] = Q K^T   8 MMAs per 8-key column tile, K^T fragments by
//                               ldmatrix from the key rows
//   online softmax per head     block max / sum over a row's 4 lanes
//   O [head][128] += P V        P rounded to bf16 straight from the S
//                               accumulators as the A fragment (the running sum
//                               adds the rounded weights, so the output stays a
//                               convex combination of the values); V fragments
//                               by ldmatrix.trans
// The warps merge (max, sum, O) in shared memory. A token whose context fits
// one chunk is finished there (divided by the sum, bf16 out); otherwise the CTA
// writes the chunk's (max, sum) and unnormalised O, and k_attn_combine (one
// CTA of 16 warps per (token, head), launched with programmatic dependent
// launch) rescales the chunks to their common max and divides by the summed
// weights.
// HBM-bound at long contexts: 512 bytes of key and value per cached row and kv
// head (2 KB per row at 4 kv heads).
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "flint_moe.h"
#include "common.cuh"

namespace flint {
namespace {

constexpr int kDh = 128;
constexpr int kMaxGroup = 8;          // query heads per kv head in one MMA tile
constexpr int kWarps = 4;
constexpr int kBlock = 16;            // keys per block
constexpr int kStages = 3;
constexpr int kRow = kDh + 8;         // padded shared-memory row (elements)
constexpr int kStageElems = 2 * kBlock * kRow;              // key rows, then value rows
constexpr int kSmemBytes = kWarps * kStages * kStageElems * 2;  // 104,448
constexpr int kChunkQuantum = kWarps * kBlock;              // 64 keys
constexpr int kCtaSlots = 2 * 148;    // resident CTAs: 2 per SM on 148 SMs
constexpr int kMaxLen = 1 << 30;      // context rows per token (chunk arithmetic stays in int)

struct Params {
  const uint16_t* q;        // [T][Hq][128]
  const uint16_t* k;        // [rows][Hkv][128]
  const uint16_t* v;
  const int64_t* start;     // [T]
  const int32_t* len;       // [T]
  float* ml;                // [T][Hkv][n_chunks][8][2]: chunk max (log2 units), sum
  float* po;                // [T][Hkv][n_chunks][8][128]: unnormalised O
  uint16_t* out;            // [T][Hq][128]
  int32_t* status;
  long long rows;
  int T, Hq, Hkv, group, chunk, n_chunks, max_len;
  float scale_log2;         // scale * log2(e)
};

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ float lo_bf16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void ldsm_x4(const void* p, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_addr(p)));
}
__device__ __forceinline__ void ldsm_x4_t(const void* p, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_addr(p)));
}
// c += A B with A rows 8..15 zero (a1 = a3 = 0)
__device__ __forceinline__ void mma_top(float (&c)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
// 16-byte global -> shared copy; src_bytes 0 fills zeros
__device__ __forceinline__ void cp16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// The token's valid context length: len[t] clamped to [0, max_len] and to rows
// that exist; a range outside the cache is dropped (zeros out). Both kernels
// apply the same rule; the partial kernel records FLINT_DEVCHECK_INDEX.
__device__ __forceinline__ int token_len(const Params& p, int t, long long& base, bool record) {
  base = p.start[t];
  int L = p.len[t];
  bool bad = false;
  if (L > p.max_len) {
    L = p.max_len;
    bad = true;
  }
  if (L < 0 || base < 0 || base + L > p.rows) {
    L = 0;
    bad = true;
  }
  if (bad && record && p.status != nullptr) atomicOr(p.status, FLINT_DEVCHECK_INDEX);
  return L;
}

__global__ void __launch_bounds__(kWarps * 32, 2) k_attn_partial(Params p) {
  extern __shared__ __align__(16) uint16_t smem[];
  __shared__ float s_m[kWarps][kMaxGroup], s_l[kWarps][kMaxGroup];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int chunk_id = blockIdx.x, g = blockIdx.y, t = blockIdx.z;
  long long base;
  const int L = token_len(p, t, base, chunk_id == 0 && g == 0 && threadIdx.x == 0);
  const int c0 = chunk_id * p.chunk;
  pdl_trigger();
  if (c0 >= L && !(chunk_id == 0 && p.n_chunks == 1)) return;  // past the context (single chunk: write zeros)
  const int c1 = min(L, c0 + p.chunk);
  const int per_warp = p.chunk / kWarps;
  const int w0 = min(c1, c0 + warp * per_warp), w1 = min(c1, w0 + per_warp);
  const int gq = lane >> 2, t4 = lane & 3;
  const bool row_live = gq < p.group;
  // Q fragments of head row gq: k-step ks covers dims 16ks .. 16ks + 15
  uint32_t qa0[8], qa2[8];
  {
    const uint16_t* qh = p.q + (static_cast<size_t>(t) * p.Hq + g * p.group + (row_live ? gq : 0)) * kDh;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qa0[ks] = row_live ? __ldg(reinterpret_cast<const uint32_t*>(qh + 16 * ks + 2 * t4)) : 0u;
      qa2[ks] = row_live ? __ldg(reinterpret_cast<const uint32_t*>(qh + 16 * ks + 8 + 2 * t4)) : 0u;
    }
  }
  float m = -INFINITY, l = 0.f;  // head row gq, replicated over the row's 4 lanes
  float o[16][2];
#pragma unroll
  for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = 0.f;
  uint16_t* ring = smem + warp * kStages * kStageElems;
  const int n_blocks = (w1 - w0 + kBlock - 1) / kBlock;
  auto load_block = [&](int b) {
    uint16_t* st = ring + (b % kStages) * kStageElems;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = lane + 32 * i, r = c >> 4, q16 = c & 15;
      const int key = w0 + b * kBlock + r;
      const bool in = key < w1;
      const size_t row = (static_cast<size_t>(base + (in ? key : w0)) * p.Hkv + g) * kDh + 8 * q16;
      cp16(st + r * kRow + 8 * q16, p.k + row, in ? 16 : 0);
      cp16(st + (kBlock + r) * kRow + 8 * q16, p.v + row, in ? 16 : 0);
    }
  };
  // prologue: blocks 0 .. kStages-2 in flight (an empty group keeps the count)
#pragma unroll
  for (int b = 0; b < kStages - 1; ++b) {
    if (b < n_blocks) load_block(b);
    cp_commit();
  }
  for (int b = 0; b < n_blocks; ++b) {
    if (b + kStages - 1 < n_blocks) load_block(b + kStages - 1);
    cp_commit();
    cp_wait<kStages - 1>();
    __syncwarp();
    const uint16_t* kr = ring + (b % kStages) * kStageElems;
    const uint16_t* vr = kr + kBlock * kRow;
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
    {
      // x4 matrices: (keys 0-7, dims +0..7), (keys 0-7, +8..15), (keys 8-15, +0..7), (keys 8-15, +8..15)
      const int mr = (lane & 7) + ((lane >> 4) << 3), mc = ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t b00, b01, b10, b11;
        ldsm_x4(kr + mr * kRow + 16 * ks + mc, b00, b01, b10, b11);
        mma_top(s0, qa0[ks], qa2[ks], b00, b01);
        mma_top(s1, qa0[ks], qa2[ks], b10, b11);
      }
    }
    // the lane holds keys 2t4, 2t4+1 (s0) and 8+2t4, 9+2t4 (s1) of head row gq
    const int kb = w0 + b * kBlock;
    float sc[4] = {s0[0] * p.scale_log2, s0[1] * p.scale_log2, s1[0] * p.scale_log2, s1[1] * p.scale_log2};
    if (kb + kBlock > w1) {
      const int kidx[4] = {2 * t4, 2 * t4 + 1, 8 + 2 * t4, 9 + 2 * t4};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (kb + kidx[j] >= w1) sc[j] = -INFINITY;
    }
    float bm = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
    const float m_new = fmaxf(m, bm);  // finite: every block holds at least one key
    const float alpha = exp2f(m - m_new);
    const uint32_t pa0 = pack_bf16x2_rn(exp2f(sc[0] - m_new), exp2f(sc[1] - m_new));
    const uint32_t pa2 = pack_bf16x2_rn(exp2f(sc[2] - m_new), exp2f(sc[3] - m_new));
    float ps = (lo_bf16(pa0) + hi_bf16(pa0)) + (lo_bf16(pa2) + hi_bf16(pa2));
    ps += __shfl_xor_sync(0xffffffffu, ps, 1);
    ps += __shfl_xor_sync(0xffffffffu, ps, 2);
    l = fmaf(l, alpha, ps);
    m = m_new;
    {
      // x4.trans matrices: (keys 0-7, dims 8j..), (keys 8-15, 8j..), (keys 0-7, 8j+8..), (keys 8-15, 8j+8..)
      const int vrow = (lane & 7) + ((lane >> 3) & 1) * 8, vcol = (lane >> 4) * 8;
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        uint32_t b0a, b1a, b0b, b1b;
        ldsm_x4_t(vr + vrow * kRow + 8 * j + vcol, b0a, b1a, b0b, b1b);
        float c0a[4] = {o[j][0] * alpha, o[j][1] * alpha, 0.f, 0.f};
        float c0b[4] = {o[j + 1][0] * alpha, o[j + 1][1] * alpha, 0.f, 0.f};
        mma_top(c0a, pa0, pa2, b0a, b1a);
        mma_top(c0b, pa0, pa2, b0b, b1b);
        o[j][0] = c0a[0];
        o[j][1] = c0a[1];
        o[j + 1][0] = c0b[0];
        o[j + 1][1] = c0b[1];
      }
    }
    __syncwarp();
  }
  cp_wait<0>();
  __syncwarp();
  // the warp's (m, l, O) -> shared memory; O into the warp's own ring
  float* s_o = reinterpret_cast<float*>(ring);  // [8][128] fp32 = 4 KB of the warp's 26 KB
  if (t4 == 0) {
    s_m[warp][gq] = m;
    s_l[warp][gq] = l;
  }
#pragma unroll
  for (int j = 0; j < 16; ++j)
    *reinterpret_cast<float2*>(s_o + gq * kDh + 8 * j + 2 * t4) = make_float2(o[j][0], o[j][1]);
  __syncthreads();
  // merge the warps: thread d owns dimension d of every head
  const int d = threadIdx.x;
  const bool single = p.n_chunks == 1;
  const size_t tgc = (static_cast<size_t>(t) * p.Hkv + g) * p.n_chunks + chunk_id;
  for (int h = 0; h < p.group; ++h) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, s_m[w][h]);
    float lsum = 0.f, acc = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float f = s_m[w][h] == -INFINITY ? 0.f : exp2f(s_m[w][h] - M);
      lsum = fmaf(s_l[w][h], f, lsum);
      acc = fmaf(reinterpret_cast<const float*>(smem + w * kStages * kStageElems)[h * kDh + d], f, acc);
    }
    if (single) {
      const float r = lsum > 0.f ? acc / lsum : 0.f;
      const __nv_bfloat16 bv = __float2bfloat16_rn(r);
      p.out[(static_cast<size_t>(t) * p.Hq + g * p.group + h) * kDh + d] = *reinterpret_cast<const uint16_t*>(&bv);
    } else {
      if (d == 0) *reinterpret_cast<float2*>(p.ml + (tgc * kMaxGroup + h) * 2) = make_float2(M, lsum);
      p.po[(tgc * kMaxGroup + h) * kDh + d] = acc;
    }
  }
}

// One CTA of 16 warps per (token, head). Warp w takes chunks w, w + 16, ...
// eight at a time, all eight chunks' loads issued before any is used (one
// round trip for up to 128 chunks), merged with a running max; lane l holds
// dimensions 4l .. 4l + 3. The warps' (max, sum, O) then meet in shared memory.
constexpr int kCombineWarps = 16;
constexpr int kCombineBatch = 8;

__global__ void __launch_bounds__(kCombineWarps * 32) k_attn_combine(Params p) {
  __shared__ float s_m[kCombineWarps], s_l[kCombineWarps];
  __shared__ __align__(16) float s_acc[kCombineWarps][kDh];
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = blockIdx.x, t = blockIdx.y;
  const int g = h / p.group, hh = h % p.group;
  long long base;
  const int L = token_len(p, t, base, false);
  const int nc = (L + p.chunk - 1) / p.chunk;
  const size_t tg = (static_cast<size_t>(t) * p.Hkv + g) * p.n_chunks;
  float M = -INFINITY, lsum = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c0 = warp; c0 < nc; c0 += kCombineWarps * kCombineBatch) {
    float2 mlv[kCombineBatch];
    float4 ov[kCombineBatch];
#pragma unroll
    for (int i = 0; i < kCombineBatch; ++i) {
      const int c = c0 + i * kCombineWarps;
      if (c < nc) {
        const size_t r = (tg + c) * kMaxGroup + hh;
        mlv[i] = __ldcg(reinterpret_cast<const float2*>(p.ml + r * 2));
        ov[i] = __ldcg(reinterpret_cast<const float4*>(p.po + r * kDh) + lane);
      } else {
        mlv[i] = make_float2(-INFINITY, 0.f);
        ov[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    float mb = M;
#pragma unroll
    for (int i = 0; i < kCombineBatch; ++i) mb = fmaxf(mb, mlv[i].x);
    if (mb == -INFINITY) continue;  // nothing in this batch or before it
    const float fo = M == -INFINITY ? 0.f : exp2f(M - mb);
    lsum *= fo;
    acc.x *= fo;
    acc.y *= fo;
    acc.z *= fo;
    acc.w *= fo;
#pragma unroll
    for (int i = 0; i < kCombineBatch; ++i) {
      const float f = mlv[i].x == -INFINITY ? 0.f : exp2f(mlv[i].x - mb);
      lsum = fmaf(mlv[i].y, f, lsum);
      acc.x = fmaf(ov[i].x, f, acc.x);
      acc.y = fmaf(ov[i].y, f, acc.y);
      acc.z = fmaf(ov[i].z, f, acc.z);
      acc.w = fmaf(ov[i].w, f, acc.w);
    }
    M = mb;
  }
  if (lane == 0) {
    s_m[warp] = M;
    s_l[warp] = lsum;
  }
  *reinterpret_cast<float4*>(&s_acc[warp][4 * lane]) = acc;
  __syncthreads();
  if (threadIdx.x >= kDh) return;
  const int d = threadIdx.x;
  float Mx = -INFINITY;
#pragma unroll
  for (int w = 0; w < kCombineWarps; ++w) Mx = fmaxf(Mx, s_m[w]);
  float tot = 0.f, num = 0.f;
#pragma unroll
  for (int w = 0; w < kCombineWarps; ++w) {
    const float f = s_m[w] == -INFINITY ? 0.f : exp2f(s_m[w] - Mx);
    tot = fmaf(s_l[w], f, tot);
    num = fmaf(s_acc[w][d], f, num);
  }
  const __nv_bfloat16 bv = __float2bfloat16_rn(tot > 0.f ? num / tot : 0.f);
  p.out[(static_cast<size_t>(t) * p.Hq + h) * kDh + d] = *reinterpret_cast<const uint16_t*>(&bv);
}

// Chunk length (a multiple of 64 keys) for max_len: about kCtaSlots CTAs over
// the T * Hkv (token, kv head) pairs, one chunk when those already fill them.
int pick_chunk(int T, int Hkv, int max_len) {
  const long long pairs = static_cast<long long>(T) * Hkv;
  long long splits = (kCtaSlots + pairs / 2) / pairs;  // nearest whole number of chunks per pair
  const long long quanta = (max_len + kChunkQuantum - 1) / kChunkQuantum;
  if (splits > quanta) splits = quanta;
  if (splits < 1) splits = 1;
  const long long per = (quanta + splits - 1) / splits;
  return static_cast<int>(per * kChunkQuantum);
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace
}  // namespace flint

using namespace flint;

extern "C" size_t flint_decode_attention_workspace_bytes(int32_t T, int32_t n_kv_heads, int32_t max_len) {
  if (T < 1 || n_kv_heads < 1 || max_len < 1 || max_len > kMaxLen) return 0;
  const int chunk = pick_chunk(T, n_kv_heads, max_len);
  const long long nch = (max_len + chunk - 1) / chunk;
  if (nch <= 1) return 0;
  const size_t units = static_cast<size_t>(T) * n_kv_heads * nch * kMaxGroup;
  return round256(units * 2 * sizeof(float)) + round256(units * kDh * sizeof(float));
}

extern "C" int flint_decode_attention(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                                      int64_t n_rows, const int64_t* start, const int32_t* len, int32_t T,
                                      int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int32_t max_len,
                                      float scale, uint16_t* out, void* workspace, size_t workspace_bytes,
                                      int32_t* status, void* stream) {
  if (head_dim != kDh) return flint_fail_external(FLINT_ERR_UNSUPPORTED_SHAPE, "head_dim must be 128");
  if (T < 0 || n_q_heads < 1 || n_kv_heads < 1 || n_rows < 0 || max_len < 0 || !(scale > 0.f))
    return flint_fail_external(FLINT_ERR_INVALID_ARG, "flint_decode_attention: bad sizes");
  if (n_q_heads % n_kv_heads != 0 || n_q_heads / n_kv_heads > kMaxGroup)
    return flint_fail_external(FLINT_ERR_UNSUPPORTED_SHAPE, "n_q_heads / n_kv_heads must be an integer <= 8");
  if (T > 65535 || n_kv_heads > 65535)
    return flint_fail_external(FLINT_ERR_UNSUPPORTED_SHAPE, "at most 65535 tokens and kv heads");
  if (max_len > kMaxLen) return flint_fail_external(FLINT_ERR_UNSUPPORTED_SHAPE, "max_len above 2^30 rows");
  if (T == 0) return FLINT_OK;
  if (!q || !out || !start || !len || (n_rows > 0 && (!k_cache || !v_cache)))
    return flint_fail_external(FLINT_ERR_INVALID_ARG, "flint_decode_attention: NULL pointer");
  const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k_cache) |
                        reinterpret_cast<uintptr_t>(v_cache) | reinterpret_cast<uintptr_t>(out) |
                        reinterpret_cast<uintptr_t>(workspace);
  if (mis & 15u) return flint_fail_external(FLINT_ERR_MISALIGNED, "flint_decode_attention: misaligned pointer");
  const int ml_eff = max_len < 1 ? 1 : max_len;
  Params p{};
  p.q = q;
  p.k = k_cache;
  p.v = v_cache;
  p.start = start;
  p.len = len;
  p.out = out;
  p.status = status;
  p.rows = n_rows;
  p.T = T;
  p.Hq = n_q_heads;
  p.Hkv = n_kv_heads;
  p.group = n_q_heads / n_kv_heads;
  p.max_len = max_len;
  p.chunk = pick_chunk(T, n_kv_heads, ml_eff);
  p.n_chunks = (ml_eff + p.chunk - 1) / p.chunk;
  p.scale_log2 = scale * 1.4426950408889634f;
  const size_t need = flint_decode_attention_workspace_bytes(T, n_kv_heads, ml_eff);
  if (need > 0) {
    if (workspace == nullptr || workspace_bytes < need)
      return flint_fail_external(FLINT_ERR_WORKSPACE, "flint_decode_attention: workspace too small");
    const size_t units = static_cast<size_t>(T) * n_kv_heads * p.n_chunks * kMaxGroup;
    p.ml = static_cast<float*>(workspace);
    p.po = reinterpret_cast<float*>(static_cast<char*>(workspace) + round256(units * 2 * sizeof(float)));
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  {
    const cudaError_t ea = flint_ensure_smem(reinterpret_cast<const void*>(k_attn_partial));
    if (ea != cudaSuccess) return flint_fail_external(FLINT_ERR_CUDA, cudaGetErrorString(ea));
  }
  k_attn_partial<<<dim3(p.n_chunks, n_kv_heads, T), kWarps * 32, kSmemBytes, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return flint_fail_external(FLINT_ERR_CUDA, cudaGetErrorString(e));
  if (p.n_chunks > 1) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(n_q_heads, T);
    cfg.blockDim = dim3(kCombineWarps * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k_attn_combine, p);
    if (e != cudaSuccess) return flint_fail_external(FLINT_ERR_CUDA, cudaGetErrorString(e));
  }
  return FLINT_OK;
}
