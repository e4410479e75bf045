// flint_moe.cu -- packer, debug kernels and the C ABI of libflint_moe.so (see
// include/flint_moe.h). The layer kernels are in layer_kernels.cuh: per layer
// k_route -> k_gateup -> k_down, chained with programmatic dependent launch on
// the caller's stream. The packer quantises and lays out weights (fp32 recipe,
// bit-exact against the CPU oracle).

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <string>

#include "fused_layer.cuh"
#include "mma_path.cuh"
#include "tok1.cuh"
#include "tokn.cuh"
#include "lmhead.cuh"

#include <cudaTypedefs.h>

namespace flint {

// ======================================================================= kernels
// ----------------------------------------------------------------- packer
// Per-matrix amax (as uint bits of non-negative floats) and non-finite check.
template <bool BF16IN>
__global__ void k_pack_amax(const void* w, long long per_mat, unsigned* amax_bits, int* status) {
  const int mat = blockIdx.y;
  float m = 0.f;
  bool bad = false;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < per_mat;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long gi = static_cast<long long>(mat) * per_mat + i;
    const float v = BF16IN ? bf16_bits_to_f32(static_cast<const uint16_t*>(w)[gi])
                           : static_cast<const float*>(w)[gi];
    if (!isfinite(v)) bad = true;
    else m = fmaxf(m, fabsf(v));
  }
  if (bad) atomicOr(status, FLINT_DEVCHECK_NONFINITE);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(&amax_bits[mat], __float_as_uint(m));
}

__device__ __forceinline__ uint32_t f32_to_e4m3(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.f), "f"(v));
  return r & 0xFFu;
}
// Two values -> one byte of E2M1 codes, `lo` in the low nibble.
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n .reg .b8 b;\n cvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n cvt.u32.u8 %0, b;\n}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r & 0xFFu;
}

// One thread per 16-element block: the recipe's fp32 steps, then the layout.
template <bool BF16IN>
__global__ void k_pack_quant(const void* w, int d, int I, long long n_blocks, long long cpe, long long spe,
                             const unsigned* amax_bits, uint8_t* codes, uint8_t* scales, float* ts) {
  const long long gb = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  if (gb >= n_blocks) return;
  const long long per_mat = static_cast<long long>(I) * d;
  const long long blocks_per_mat = per_mat / 16;
  const int mat = static_cast<int>(gb / blocks_per_mat);
  const long long bi = gb % blocks_per_mat;
  const int e = mat / 3, m = mat % 3;
  const int cols = (m < 2) ? d : I;
  const int r = static_cast<int>(bi / (cols / 16)), b = static_cast<int>(bi % (cols / 16));
  float v[16];
  const long long base = static_cast<long long>(mat) * per_mat + static_cast<long long>(r) * cols + 16LL * b;
  if (BF16IN) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(w) + base);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint4 u = src[q];
      const uint32_t ww[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[8 * q + 2 * i] = bf16_bits_to_f32(ww[i] & 0xFFFFu);
        v[8 * q + 2 * i + 1] = __uint_as_float(ww[i] & 0xFFFF0000u);
      }
    }
  } else {
    const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(w) + base);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 f = src[q];
      v[4 * q] = f.x;
      v[4 * q + 1] = f.y;
      v[4 * q + 2] = f.z;
      v[4 * q + 3] = f.w;
    }
  }
  const float amax = __uint_as_float(amax_bits[mat]);
  const float s_t = (amax > 0.f) ? __fdiv_rn(amax, 2688.f) : 1.f;
  float amax_b = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax_b = fmaxf(amax_b, fabsf(v[i]));
  const uint32_t sb = f32_to_e4m3(__fdiv_rn(__fdiv_rn(amax_b, 6.f), s_t));
  const float dec = e4m3x2_to_f32x2(sb).x;
  const float denom = __fmul_rn(dec, s_t);
  uint32_t lo = 0, hi = 0;
  if (denom != 0.f) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      lo |= f32x2_to_e2m1x2(__fdiv_rn(v[2 * i], denom), __fdiv_rn(v[2 * i + 1], denom)) << (8 * i);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      hi |= f32x2_to_e2m1x2(__fdiv_rn(v[8 + 2 * i], denom), __fdiv_rn(v[8 + 2 * i + 1], denom)) << (8 * i);
  }
  long long co, so;
  if (m == 0) {
    co = static_cast<long long>(r) * d + 8LL * b;
    so = static_cast<long long>(r) * (d / 8) + b;
  } else if (m == 1) {
    co = static_cast<long long>(r) * d + d / 2 + 8LL * b;
    so = static_cast<long long>(r) * (d / 8) + d / 16 + b;
  } else {
    co = static_cast<long long>(I) * d + static_cast<long long>(r) * (I / 2) + 8LL * b;
    so = static_cast<long long>(I) * d / 8 + static_cast<long long>(r) * (I / 16) + b;
  }
  *reinterpret_cast<uint2*>(codes + e * cpe + co) = make_uint2(lo, hi);
  scales[e * spe + so] = static_cast<uint8_t>(sb);
  if (r == 0 && b == 0) ts[mat] = s_t;
}

// One dense matrix [rows][cols], row-major planes: codes [rows][cols/2],
// scales [rows][cols/16], one tensor scale (the same recipe as k_pack_quant).
template <bool BF16IN>
__global__ void k_pack_dense_quant(const void* w, long long rows, int cols, const unsigned* amax_bits, uint8_t* codes,
                                   uint8_t* scales, float* ts) {
  const long long gb = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  const long long n_blocks = rows * (cols / 16);
  if (gb >= n_blocks) return;
  float v[16];
  if (BF16IN) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(w) + 16 * gb);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint4 u = src[q];
      const uint32_t ww[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[8 * q + 2 * i] = bf16_bits_to_f32(ww[i] & 0xFFFFu);
        v[8 * q + 2 * i + 1] = __uint_as_float(ww[i] & 0xFFFF0000u);
      }
    }
  } else {
    const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(w) + 16 * gb);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 f = src[q];
      v[4 * q] = f.x;
      v[4 * q + 1] = f.y;
      v[4 * q + 2] = f.z;
      v[4 * q + 3] = f.w;
    }
  }
  const float amax = __uint_as_float(amax_bits[0]);
  const float s_t = (amax > 0.f) ? __fdiv_rn(amax, 2688.f) : 1.f;
  float amax_b = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax_b = fmaxf(amax_b, fabsf(v[i]));
  const uint32_t sb = f32_to_e4m3(__fdiv_rn(__fdiv_rn(amax_b, 6.f), s_t));
  const float dec = e4m3x2_to_f32x2(sb).x;
  const float denom = __fmul_rn(dec, s_t);
  uint32_t lo = 0, hi = 0;
  if (denom != 0.f) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      lo |= f32x2_to_e2m1x2(__fdiv_rn(v[2 * i], denom), __fdiv_rn(v[2 * i + 1], denom)) << (8 * i);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      hi |= f32x2_to_e2m1x2(__fdiv_rn(v[8 + 2 * i], denom), __fdiv_rn(v[8 + 2 * i + 1], denom)) << (8 * i);
  }
  *reinterpret_cast<uint2*>(codes + 8 * gb) = make_uint2(lo, hi);
  scales[gb] = static_cast<uint8_t>(sb);
  if (gb == 0) ts[0] = s_t;
}

// bf16 weights in the same expert-major row order (16-byte vectors).
__global__ void k_pack_bf16(const uint16_t* w, int d, int I, long long n_vec, uint16_t* out) {
  const long long gv = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  if (gv >= n_vec) return;
  const long long per_mat = static_cast<long long>(I) * d;
  const long long vec_per_mat = per_mat / 8;
  const int mat = static_cast<int>(gv / vec_per_mat);
  const long long vi = gv % vec_per_mat;
  const int e = mat / 3, m = mat % 3;
  const int cols = (m < 2) ? d : I;
  const int r = static_cast<int>(vi / (cols / 8)), c8 = static_cast<int>(vi % (cols / 8));
  const uint4 val = reinterpret_cast<const uint4*>(w + static_cast<long long>(mat) * per_mat)[vi];
  long long o = static_cast<long long>(e) * 3 * per_mat;
  if (m == 0) o += static_cast<long long>(r) * 2 * d + 8LL * c8;
  else if (m == 1) o += static_cast<long long>(r) * 2 * d + d + 8LL * c8;
  else o += 2LL * I * d + static_cast<long long>(r) * I + 8LL * c8;
  *reinterpret_cast<uint4*>(out + o) = val;
}

// Decoded e2m1*e4m3 products of rows of one expert matrix, through the same
// decode routines the layer kernels use. One thread per 32-element vector.
__global__ void k_debug_dequant(const uint8_t* codes, const uint8_t* scales, int K, long long rows,
                                float* out) {
  const long long gv = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  const int vpr = K / 32;
  if (gv >= rows * vpr) return;
  const long long r = gv / vpr;
  const int v = static_cast<int>(gv % vpr);
  const uint4 c = *reinterpret_cast<const uint4*>(codes + r * (K / 2) + v * 16);
  const uint32_t s2 = *reinterpret_cast<const uint16_t*>(scales + r * (K / 16) + v * 2);
  const float2 s = e4m3x2_to_f32x2(s2);
  const uint32_t words[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int wi = 0; wi < 4; ++wi) {
    uint32_t q[4];
    e2m1x8_to_f16x2(words[wi], q);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&q[i]));
      const float sc = (wi < 2) ? s.x : s.y;
      out[r * K + v * 32 + wi * 8 + 2 * i] = f.x * sc;
      out[r * K + v * 32 + wi * 8 + 2 * i + 1] = f.y * sc;
    }
  }
}

// The tensor-core path's NVFP4 decode (dequant_slice_tmem) on one tile of 128
// rows x 256 K: the tile is staged the way its TMA copy lands (code rows of
// 128 bytes with the 128-byte swizzle, then 16 scale bytes per row), decoded
// into tensor memory by warps 8..15 exactly as in k_mma_ffn, read back with
// tcgen05.ld by warps 4..7 (lanes 32*(w%4)..) and written as fp32. Column c of
// the tile's 128 tensor-memory columns holds K elements 2c, 2c+1 as f16x2.
// Grid (row tiles, K tiles); `codes`/`scales` point at the matrix's first row.
__global__ void __launch_bounds__(512, 1) k_debug_decode_tmem(const uint8_t* codes, const uint8_t* scales, int K,
                                                              int k0, float* out, int ldo) {
  __shared__ __align__(1024) uint8_t raw[kMmaRawBytes];
  __shared__ uint32_t s_tmem;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long r0 = 128LL * blockIdx.x;
  const int kb = k0 + 256 * blockIdx.y;
  for (int i = tid; i < 128 * 8; i += blockDim.x) {  // 16-byte code chunks, swizzled as TMA writes them
    const int r = i >> 3, c = i & 7;
    *reinterpret_cast<uint4*>(raw + r * 128 + ((c ^ (r & 7)) << 4)) =
        *reinterpret_cast<const uint4*>(codes + (r0 + r) * (K / 2) + kb / 2 + 16 * c);
  }
  for (int i = tid; i < 128; i += blockDim.x)
    *reinterpret_cast<uint4*>(raw + 128 * 128 + 16 * i) =
        *reinterpret_cast<const uint4*>(scales + (r0 + i) * (K / 16) + kb / 16);
  if (warp == 1) tmem_alloc(&s_tmem, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  if (warp >= 8)
    for (int sub = 0; sub < 4; ++sub) dequant_slice_tmem(raw, sub, tmem + 32u * sub, warp & 3, (warp - 8) >> 2, lane);
  tmem_wait_st();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp >= 4 && warp < 8) {
    const int row = 32 * (warp & 3) + lane;
    for (int c0 = 0; c0 < 128; c0 += 16) {
      float v[16];
      tmem_ld16(tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + static_cast<uint32_t>(c0), v);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint32_t w = __float_as_uint(v[i]);
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w));
        float* o = out + (r0 + row) * ldo + 256 * blockIdx.y + 2 * (c0 + i);
        o[0] = f.x;
        o[1] = f.y;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// The persistent kernel's register-fragment decode (tc_segment) on tiles of
// 16 rows x 128 K, extracted through the MMA itself: in step q, B column n is
// one-hot on the logical k that the segment's K permutation gives physical
// element 8q + n, so D[row][n] = A[row][8q + n], the decoded weight of that
// element (exact in f16, multiplied by 1 and accumulated in f32). One warp per
// tile; grid (row tiles, K tiles).
__global__ void __launch_bounds__(32) k_debug_decode_frag(const uint8_t* codes, const uint8_t* scales, int K, int k0,
                                                          float* out, int ldo) {
  const int lane = threadIdx.x, g = lane >> 2, t = lane & 3;
  const long long r0 = 16LL * blockIdx.x;
  const int kb = k0 + 128 * blockIdx.y;
  const uint4 ra = *reinterpret_cast<const uint4*>(codes + (r0 + g) * (K / 2) + kb / 2 + 16 * t);
  const uint4 rb = *reinterpret_cast<const uint4*>(codes + (r0 + g + 8) * (K / 2) + kb / 2 + 16 * t);
  const uint32_t sa2 = *reinterpret_cast<const uint16_t*>(scales + (r0 + g) * (K / 16) + kb / 16 + 2 * t);
  const uint32_t sb2 = *reinterpret_cast<const uint16_t*>(scales + (r0 + g + 8) * (K / 16) + kb / 16 + 2 * t);
  for (int q = 0; q < 16; ++q) {
    // this lane holds B rows k = 2t, 2t+1 (b[2j]) and 2t+8, 2t+9 (b[2j+1]) of
    // column g; physical element p = 32t' + 4j + 2h + e sits in b[2j+h], half e,
    // of the lanes with t = t'
    const int p = 8 * q + g, tp = p >> 5, j = (p & 31) >> 2, h = (p >> 1) & 1, e = p & 1;
    uint32_t b[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) b[i] = (tp == t && i == 2 * j + h) ? (e ? 0x3C000000u : 0x00003C00u) : 0u;
    float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
    tc_segment(c0, c1, ra, rb, sa2, sb2, b);
    // c[0..1]: row g, columns 2t, 2t+1; c[2..3]: row g + 8
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = g + 8 * (i >> 1), col = 2 * t + (i & 1);
      out[(r0 + row) * ldo + 128 * blockIdx.y + 8 * q + col] = c0[i] + c1[i];
    }
  }
}

// One of the grouping routines on given ids (debug entry flint_debug_group):
// impl 0 the CTA grouping of the persistent kernel and the tensor-core path
// (T <= 128), 1 the warp grouping of the three-kernel path (T*k <= 64), 2 its
// CTA grouping (T <= 32). One CTA of 512 threads; outputs as int arrays.
// counts[0] (routed experts in use) from counts[1] (active experts).
__global__ void k_debug_routed_count(int* counts, int S) { counts[0] = counts[1] - S; }

__global__ void __launch_bounds__(512) k_debug_group(const int* ids, int T, int k, int E, int S, int impl, int* act,
                                                     int* off, int* pair, int* counts, int* status) {
  __shared__ int s_ids[kMmaMaxTokens * kMaxTopK];
  __shared__ __align__(8) uint8_t s_scratch[20 * kMaxExperts];
  __shared__ Grouping g;
  __shared__ RouteDesc dsc;
  const int tid = threadIdx.x;
  for (int i = tid; i < T * k; i += blockDim.x) s_ids[i] = ids[i];
  __syncthreads();
  if (impl == 0) {
    cta_grouping(s_ids, T, k, E, S, act, off, pair, counts, counts + 1, s_scratch, status);
    return;
  }
  const int* a;
  const int* o;
  const unsigned short* pr;
  int n_active, n_routed;
  if (impl == 1) {
    if (tid < 32) warp_grouping(s_ids, T, k, E, S, &dsc, tid, status);
    __syncthreads();
    a = dsc.act;
    o = dsc.off;
    pr = dsc.pair;
    n_active = dsc.n_active;
    n_routed = dsc.n_routed;
  } else {
    build_grouping(g, s_ids, T, k, E, S, status);
    a = g.act;
    o = g.off;
    pr = g.pair;
    n_active = g.n_active;
    n_routed = g.n_routed;
  }
  for (int i = tid; i < n_active; i += blockDim.x) act[i] = a[i];
  for (int i = tid; i <= n_active; i += blockDim.x) off[i] = o[i];
  for (int i = tid; i < o[n_active]; i += blockDim.x) pair[i] = pr[i];
  if (tid == 0) {
    counts[0] = n_routed;
    counts[1] = n_active;
  }
}

// A wait on a barrier that no thread or copy ever completes: the bounded loop
// gives up after `cycles` and records FLINT_DEVCHECK_WAIT.
__global__ void k_debug_wait(int* status, long long cycles) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const long long t0 = clock64();
    while (!mbar_try_wait(&bar, 0)) {
      if (clock64() - t0 > cycles) {
        atomicOr(status, FLINT_DEVCHECK_WAIT);
        break;
      }
    }
  }
}

// ======================================================================= host side
namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

}  // namespace

// The last-error slot for the library's other translation units.
int flint_fail_external(int code, const char* msg) { return fail(code, "%s", msg); }

namespace {

int cuda_fail(cudaError_t e, const char* what) {
  // a failed launch or call also stays in the runtime's last-error slot; take
  // it out so that a later, unrelated check does not report it again
  cudaGetLastError();
  return fail(FLINT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

struct Dims {
  int d, I, E, k, S, wd;
};

int check_shape(const flint_moe_shape* s, Dims* out) {
  if (s == nullptr) return fail(FLINT_ERR_INVALID_ARG, "shape is NULL");
  const int d = s->d, I = s->inter, E = s->n_experts, k = s->top_k, S = s->n_shared;
  if (s->wdtype != FLINT_W_NVFP4 && s->wdtype != FLINT_W_BF16)
    return fail(FLINT_ERR_INVALID_ARG, "wdtype %d is not a flint_wdtype", s->wdtype);
  if (!(d == 512 || d == 1024 || d == 2048 || d == 4096))
    return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "d=%d: supported 512, 1024, 2048, 4096", d);
  if (!(I == 128 || I == 256 || I == 512 || I == 1024))
    return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "inter=%d: supported 128, 256, 512, 1024", I);
  if (E < 1 || E > kMaxExperts) return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "n_experts=%d: supported 1..%d", E, kMaxExperts);
  if (k < 1 || k > kMaxTopK || k > E) return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "top_k=%d: supported 1..min(8, E)", k);
  if (S < 0 || S > 1) return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "n_shared=%d: supported 0 or 1", S);
  *out = Dims{d, I, E, k, S, s->wdtype};
  return FLINT_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct WsLayout {
  size_t status, counter, rb_count, amax, desc, logits, tlogits, ids, gates, h, htag, tok1_part;
  size_t mma_n, mma_act, mma_off, mma_pair, xinv, hinv, xrows, hrows, y;  // tensor-core path
  size_t mma_tiles, mma_mask, mma_wpre, mma_cnt;  // its token tiles and large-T grouping scratch
  size_t total;
};

size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Token tiles of a call of up to maxT tokens: each active expert's pairs in
// runs of at most kMmaMaxTokens; at most P / kMmaMaxTokens + one per expert.
size_t mma_max_tiles(const Dims& s, int maxT) {
  const size_t P = static_cast<size_t>(maxT) * (s.k + s.S);
  return P / kMmaMaxTokens + s.E + s.S + 1;
}
constexpr size_t kCtrlBytes = 1024;

// Workspace carve-up for calls of up to maxT tokens. The first kCtrlBytes hold
// the control block: the status word (byte 0), the router's arrival counter
// (byte 4, left at zero by every call), the persistent layer kernel's launch
// generation (byte 8) and the cluster kernels' per-row-block arrival counters
// (bytes 64..127, left at zero by every call); the rest is reserved. The tagged regions start
// with a tag of 0, which no launch uses. flint_moe_workspace_init zeroes the
// whole workspace.
// Regions of the tensor-core path are laid out only when `mma` (the call takes
// that path; flint_moe_workspace_bytes reports the size with them).
WsLayout ws_layout(const Dims& s, int maxT, bool mma) {
  WsLayout w{};
  size_t o = 0;
  w.status = 0;
  w.counter = 4;
  w.rb_count = 64;
  o += kCtrlBytes;
  // the persistent kernel's tagged regions sit at offsets that do not depend
  // on the call's token count, so they only ever hold zeros or tagged words
  // of earlier launches on this workspace (older tags)
  w.tlogits = o;
  o += al256(sizeof(unsigned long long) * kLogitReplicas * static_cast<size_t>(kFusedMaxTokens) * s.E);
  w.htag = o;
  o += al256(sizeof(unsigned long long) * static_cast<size_t>(kFusedMaxTokens) * (s.k + s.S) * s.I);
  w.tok1_part = o;  // the cluster kernels' gated partial outputs [min(T, 8) * (k+S)][d]
  o += al256(sizeof(float) * static_cast<size_t>(maxT < kTnMaxTokens ? maxT : kTnMaxTokens) * (s.k + s.S) * s.d);
  w.amax = o;
  o += al256(sizeof(float) * (s.E + s.S) * 3);
  w.desc = o;
  o += al256(sizeof(RouteDesc));
  w.logits = o;
  o += al256(sizeof(float) * static_cast<size_t>(maxT) * s.E);
  w.ids = o;
  o += al256(sizeof(int) * static_cast<size_t>(maxT) * s.k);
  w.gates = o;
  o += al256(sizeof(float) * static_cast<size_t>(maxT) * s.k);
  w.h = o;
  const size_t P = static_cast<size_t>(maxT) * (s.k + s.S);
  o += al256(sizeof(float) * P * s.I);
  if (!mma) {
    w.mma_n = w.mma_act = w.mma_off = w.mma_pair = w.xinv = w.hinv = w.xrows = w.hrows = w.y = 0;
    w.mma_tiles = w.mma_mask = w.mma_wpre = w.mma_cnt = 0;
    w.total = o;
    return w;
  }
  w.mma_n = o;
  o += 256;
  w.mma_act = o;
  o += al256(sizeof(int) * (s.E + s.S));
  w.mma_off = o;
  o += al256(sizeof(int) * (s.E + s.S + 1));
  w.mma_pair = o;
  o += al256(sizeof(int) * P);
  w.xinv = o;
  o += al256(sizeof(float) * P);
  w.hinv = o;
  o += al256(sizeof(float) * P);
  w.xrows = o;
  o += al256(2 * P * s.d);
  w.hrows = o;
  o += al256(2 * P * s.I);
  w.y = o;
  o += al256(sizeof(float) * P * s.d);
  // token tiles: [1 + 3 * max tiles] ints (count, then the three arrays)
  w.mma_tiles = o;
  o += al256(sizeof(int) * (1 + 3 * mma_max_tiles(s, maxT)));
  // large-T grouping (more than kMmaGroupSmallT tokens): bit masks and word
  // prefix counts [E][T/32], counts [E]
  const size_t words = maxT > kMmaGroupSmallT ? static_cast<size_t>(s.E) * ((maxT + 31) / 32) : 0;
  w.mma_mask = o;
  o += al256(sizeof(uint32_t) * words);
  w.mma_wpre = o;
  o += al256(sizeof(int) * words);
  w.mma_cnt = o;
  o += al256(sizeof(int) * (words ? s.E : 0));
  w.total = o;
  return w;
}

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

// Raise a kernel's dynamic shared-memory limit to the device's opt-in maximum,
// once per (kernel, device). The limit only bounds what a launch may request.
cudaError_t ensure_smem(const void* kern) {
  static std::mutex mu;
  static const void* done_kern[256];
  static int done_dev[256];
  static int n_done = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  for (int i = 0; i < n_done; ++i)
    if (done_kern[i] == kern && done_dev[i] == dev) return cudaSuccess;
  int optin = 0;
  e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           optin - static_cast<int>(fa.sharedSizeBytes));
  if (e == cudaSuccess && n_done < 256) {
    done_kern[n_done] = kern;
    done_dev[n_done] = dev;
    ++n_done;
  }
  return e;
}

template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                   Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Shared-memory budget of one CTA of the streaming kernels (rings + staged
// activations), below the 227 KB opt-in limit with room for static arrays.
constexpr int kSmemBudget = 200 * 1024;

void fill_common(LayerParams& p, const Dims& s, const WsLayout& w, uint8_t* ws, int T) {
  p.T = T;
  p.d = s.d;
  p.I = s.I;
  p.E = s.E;
  p.k = s.k;
  p.S = s.S;
  p.cpe = 3LL * s.I * s.d / 2;
  p.spe = 3LL * s.I * s.d / 16;
  p.status = reinterpret_cast<int*>(ws + w.status);
  p.counter = reinterpret_cast<unsigned*>(ws + w.counter);
  p.desc = reinterpret_cast<RouteDesc*>(ws + w.desc);
  p.logits = reinterpret_cast<float*>(ws + w.logits);
  p.tlogits = reinterpret_cast<unsigned long long*>(ws + w.tlogits);
  p.htag = reinterpret_cast<unsigned long long*>(ws + w.htag);
  p.ids = reinterpret_cast<int*>(ws + w.ids);
  p.gates = reinterpret_cast<float*>(ws + w.gates);
  p.h = reinterpret_cast<float*>(ws + w.h);
}

int gateup_stage_bytes(int d) {
  const int cu = (d <= 1024) ? 4 : (d == 2048 ? 2 : 1);
  return cu * (d + d / 8);
}

// Ring depths, row blocking of the down kernel and activation staging for a call.
void configure(LayerParams& p, const Dims& s, int T) {
  const int sms = num_sms();
  const int desc = static_cast<int>(sizeof(RouteDesc));
  // gate/up: stage x in shared memory when two stages per warp still fit
  p.stage_gateup = gateup_stage_bytes(s.d);
  const int ring2 = kGemvWarps * 2 * p.stage_gateup;
  const int xbytes = T * s.d * 2;
  p.x_in_smem = (desc + xbytes + ring2 <= kSmemBudget) ? 1 : 0;
  const int room_g = kSmemBudget - desc - (p.x_in_smem ? xbytes : 0);
  p.ns_gateup = room_g / (kGemvWarps * p.stage_gateup);
  if (p.ns_gateup > 4) p.ns_gateup = 4;
  if (p.ns_gateup < 2) p.ns_gateup = 2;
  // down: rows per CTA ~ d / #SMs in whole warp steps; items of up to four steps
  const int rps = 32 / (s.I / 32);
  int nb = (s.d + sms - 1) / sms;
  nb = ((nb + rps - 1) / rps) * rps;
  if (nb % 2) nb += rps;
  p.down_nb = nb;
  p.down_rb = (4 * rps < nb) ? 4 * rps : nb;
  p.stage_down = ((p.down_rb * (s.I / 2 + s.I / 16)) + 15) & ~15;
  const int ybytes = ((4 * T * (s.k + s.S) * nb) + 127) & ~127;
  const int hbytes = T * (s.k + s.S) * s.I * 4;
  const int ring2d = kGemvWarps * 2 * p.stage_down;
  p.h_in_smem = (desc + hbytes + ybytes + ring2d <= kSmemBudget) ? 1 : 0;
  const int room_d = kSmemBudget - desc - ybytes - (p.h_in_smem ? hbytes : 0);
  p.ns_down = room_d / (kGemvWarps * p.stage_down);
  if (p.ns_down > 4) p.ns_down = 4;
  if (p.ns_down < 2) p.ns_down = 2;
}

size_t gateup_smem(const LayerParams& p) {
  return sizeof(RouteDesc) + (p.x_in_smem ? static_cast<size_t>(p.T) * p.d * 2 : 0) +
         static_cast<size_t>(kGemvWarps) * p.ns_gateup * p.stage_gateup;
}
size_t down_smem(const LayerParams& p) {
  const size_t ybytes = ((sizeof(float) * static_cast<size_t>(p.T) * (p.k + p.S) * p.down_nb) + 127) & ~static_cast<size_t>(127);
  return sizeof(RouteDesc) + (p.h_in_smem ? static_cast<size_t>(p.T) * (p.k + p.S) * p.I * 4 : 0) + ybytes +
         static_cast<size_t>(kGemvWarps) * p.ns_down * p.stage_down;
}

// Configuration of the tensor-core variant of the persistent layer kernel:
// gate/up rings of 16-row x 512-column stages (two 2 KiB swizzled code boxes
// + 512 B of scales, 1 KiB-aligned), K-part sum slots for the most tiles one
// CTA can get, down stages of 16 rows; the down phase's buffers lie over
// everything after the routing descriptor. Returns the dynamic shared-memory
// bytes, or 0 if the call does not fit.
size_t configure_fused_tc(LayerParams& p, const Dims& s, int T, int sms) {
  // the kernel's balanced tile split gives each CTA at most one shared-expert tile
  if (s.S * (s.I / kTcUnits) > sms) return 0;
  const size_t a128 = 127;
  auto al = [&](size_t v) { return (v + a128) & ~a128; };
  const int rps = 32 / (s.I / 32);
  int nb = (s.d + sms - 1) / sms;
  nb = ((nb + rps - 1) / rps) * rps;
  if (nb % 2) nb += rps;
  p.down_nb = nb;
  p.down_rb = 16;
  p.stage_down = 16 * (s.I / 2 + s.I / 16);
  p.ns_gateup = 2;
  p.stage_gateup = kTcStageCodes + kTcStageScales;
  p.h_in_smem = 1;
  const long long nt_max = static_cast<long long>(std::min(s.E, T * s.k) + s.S) * (s.I / kTcUnits);
  p.tc_lt = static_cast<int>((nt_max + sms - 1) / sms) + 2;
  const int R = T * (s.k + s.S);
  const size_t head = sizeof(RouteDesc) + al(static_cast<size_t>(T) * tc_b_stride(s.d)) +
                      fused_rows_bytes((s.E + sms - 1) / sms * s.d * 2, s.E) + 1024;
  const size_t p3 = static_cast<size_t>(kFusedWarps) * p.ns_gateup * (kTcStageCodes + kTcStageScales) +
                    al(static_cast<size_t>(p.tc_lt) * 129 * 4);
  const size_t budget = 218 * 1024;
  size_t p4 = 0;
  for (p.ns_down = 2; p.ns_down >= 1; --p.ns_down) {  // one down stage per warp when two do not fit (inter 1024)
    p4 = al(sizeof(RouteDesc)) + al(static_cast<size_t>(R) * tc_b_stride(s.I)) + al(4 * static_cast<size_t>(R) * nb) +
         static_cast<size_t>(kFusedWarps) * p.ns_down * p.stage_down;
    if (p4 <= budget) break;
  }
  const size_t need = std::max(head + p3, p4);
  return (p.ns_down >= 1 && need <= budget) ? need : 0;
}

// Configuration of the persistent single-kernel layer (T <= 8): returns the
// dynamic shared-memory bytes, or 0 if the call does not fit it.
size_t configure_fused(LayerParams& p, const Dims& s, int T, bool tc) {
  const int sms = num_sms();
  if (sms > 240) return 0;  // the kernel's work split uses 32-bit products of the CTA index
  p.tc_lt = 0;
  if (tc) return configure_fused_tc(p, s, T, sms);
  p.stage_gateup = gateup_stage_bytes(s.d);
  p.ns_gateup = 2;
  const int rps = 32 / (s.I / 32);
  int nb = (s.d + sms - 1) / sms;
  nb = ((nb + rps - 1) / rps) * rps;
  if (nb % 2) nb += rps;
  p.down_nb = nb;
  p.down_rb = (4 * rps < nb) ? 4 * rps : nb;
  p.stage_down = ((p.down_rb * (s.I / 2 + s.I / 16)) + 15) & ~15;
  p.ns_down = 2;
  p.h_in_smem = 1;
  const size_t a128 = 127;
  const int R = T * (s.k + s.S);
  const size_t head = sizeof(RouteDesc) + ((static_cast<size_t>(T) * s.d * 2 + a128) & ~a128) +
                      fused_rows_bytes((s.E + sms - 1) / sms * s.d * 2, s.E);
  const size_t ybytes = ((4 * static_cast<size_t>(R) * nb) + a128) & ~a128;
  const size_t ring_d = static_cast<size_t>(kFusedWarps) * p.ns_down * p.stage_down;
  const size_t down = fused_h16_bytes(R, s.I) + ybytes + ring_d;
  const size_t budget = 210 * 1024;
  // deeper gate/up rings while they fit (the down ring takes the next 2 of
  // each warp's kMaxStages barriers)
  while (p.ns_gateup < kMaxStages - 2 && p.ns_gateup < 4 &&
         head + static_cast<size_t>(kFusedWarps) * (p.ns_gateup + 1) * p.stage_gateup <= budget)
    ++p.ns_gateup;
  const size_t ring_g = static_cast<size_t>(kFusedWarps) * p.ns_gateup * p.stage_gateup;
  const size_t work = std::max(ring_g, down);
  if (head + work > budget) return 0;
  return head + work;
}

template <int D, int I, bool TC>
cudaError_t launch_fused_di(const LayerParams& p, const FusedMaps& maps, size_t smem, cudaStream_t st) {
  auto kern = k_layer<D, I, TC>;
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms());
  cfg.blockDim = dim3(kFusedWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeCooperative;
  at[0].val.cooperative = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p, maps);
}

template <int D, bool TC>
cudaError_t launch_fused_d(const LayerParams& p, const FusedMaps& maps, size_t smem, cudaStream_t st) {
  switch (p.I) {
    case 128: return launch_fused_di<D, 128, TC>(p, maps, smem, st);
    case 256: return launch_fused_di<D, 256, TC>(p, maps, smem, st);
    case 512: return launch_fused_di<D, 512, TC>(p, maps, smem, st);
    default: return launch_fused_di<D, 1024, TC>(p, maps, smem, st);
  }
}

template <bool TC>
cudaError_t launch_fused_t(const LayerParams& p, const FusedMaps& maps, size_t smem, cudaStream_t st) {
  switch (p.d) {
    case 512: return launch_fused_d<512, TC>(p, maps, smem, st);
    case 1024: return launch_fused_d<1024, TC>(p, maps, smem, st);
    case 2048: return launch_fused_d<2048, TC>(p, maps, smem, st);
    default: return launch_fused_d<4096, TC>(p, maps, smem, st);
  }
}

cudaError_t launch_fused(const LayerParams& p, const FusedMaps* maps, size_t smem, cudaStream_t st) {
  if (maps != nullptr) return launch_fused_t<true>(p, *maps, smem, st);
  FusedMaps none;
  std::memset(&none, 0, sizeof(none));
  return launch_fused_t<false>(p, none, smem, st);
}

template <typename K>
cudaError_t launch_smem(K kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                        const LayerParams& p) {
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kern));
  if (e != cudaSuccess) return e;
  return launch(kern, grid, block, smem, st, pdl, p);
}

cudaError_t launch_route_fwd(const LayerParams& p, cudaStream_t st, bool pdl) {
  const int tasks = p.E + p.S * p.I;
  const dim3 grid((tasks + kRouteWarps - 1) / kRouteWarps), block(kRouteWarps * 32);
  const size_t smem = static_cast<size_t>(p.T) * p.d * 2;
  switch (p.d) {
    case 512: return launch_smem(k_route<512>, grid, block, smem, st, pdl, p);
    case 1024: return launch_smem(k_route<1024>, grid, block, smem, st, pdl, p);
    case 2048: return launch_smem(k_route<2048>, grid, block, smem, st, pdl, p);
    default: return launch_smem(k_route<4096>, grid, block, smem, st, pdl, p);
  }
}

cudaError_t launch_router_only(const LayerParams& p, cudaStream_t st) {
  const dim3 grid((p.E + 7) / 8, (p.T + kRouterTokens - 1) / kRouterTokens), block(256);
  switch (p.d) {
    case 512: return launch(k_router_only<512>, grid, block, 0, st, false, p);
    case 1024: return launch(k_router_only<1024>, grid, block, 0, st, false, p);
    case 2048: return launch(k_router_only<2048>, grid, block, 0, st, false, p);
    default: return launch(k_router_only<4096>, grid, block, 0, st, false, p);
  }
}

cudaError_t launch_gateup(const LayerParams& p, cudaStream_t st, bool pdl) {
  const dim3 grid(num_sms()), block(kGemvWarps * 32);
  const size_t smem = gateup_smem(p);
  switch (p.d) {
    case 512: return launch_smem(k_gateup<512>, grid, block, smem, st, pdl, p);
    case 1024: return launch_smem(k_gateup<1024>, grid, block, smem, st, pdl, p);
    case 2048: return launch_smem(k_gateup<2048>, grid, block, smem, st, pdl, p);
    default: return launch_smem(k_gateup<4096>, grid, block, smem, st, pdl, p);
  }
}

cudaError_t launch_down(const LayerParams& p, cudaStream_t st, bool pdl) {
  const dim3 grid((p.d + p.down_nb - 1) / p.down_nb), block(kGemvWarps * 32);
  const size_t smem = down_smem(p);
  switch (p.I) {
    case 128: return launch_smem(k_down<128>, grid, block, smem, st, pdl, p);
    case 256: return launch_smem(k_down<256>, grid, block, smem, st, pdl, p);
    case 512: return launch_smem(k_down<512>, grid, block, smem, st, pdl, p);
    default: return launch_smem(k_down<1024>, grid, block, smem, st, pdl, p);
  }
}

// ----------------------------------------------------------------- tensor-core path (host)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// Row-major tensor of `rank` dims (dim 0 innermost, in elements), strides of
// dims 1.. in bytes, box in elements.
int encode_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const cuuint64_t* dims,
               const cuuint64_t* strides, const cuuint32_t* box, bool swizzle128) {
  auto fn = tensor_map_encoder();
  if (fn == nullptr) return fail(FLINT_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FLINT_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return FLINT_OK;
}

// Tensor maps of one projection. gate/up: rows 2I, K = d, starting at the
// expert base; down: rows d, K = I, starting I*d (NVFP4 bytes) after it.
int mma_maps(MmaMaps* mp, const Dims& s, const flint_moe_weights* wts, bool gateup, const uint16_t* brows, int P) {
  const int K = gateup ? s.d : s.I, rows = gateup ? 2 * s.I : s.d;
  const cuuint64_t ne = static_cast<cuuint64_t>(s.E + s.S);
  int rc;
  if (s.wd == FLINT_W_NVFP4) {
    const uint8_t* codes = static_cast<const uint8_t*>(wts->packed) + (gateup ? 0 : static_cast<size_t>(s.I) * s.d);
    const uint8_t* scales = wts->block_scales + (gateup ? 0 : static_cast<size_t>(s.I) * s.d / 8);
    const cuuint64_t cdims[3] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows), ne};
    const cuuint64_t cstr[2] = {static_cast<cuuint64_t>(K / 2), 3ull * s.I * s.d / 2};
    const cuuint32_t cbox[3] = {128, 128, 1};
    if ((rc = encode_map(&mp->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, codes, cdims, cstr, cbox, true)) != FLINT_OK)
      return rc;
    const cuuint64_t sdims[3] = {static_cast<cuuint64_t>(K / 16), static_cast<cuuint64_t>(rows), ne};
    const cuuint64_t sstr[2] = {static_cast<cuuint64_t>(K / 16), 3ull * s.I * s.d / 16};
    const cuuint32_t sbox[3] = {16, 128, 1};
    if ((rc = encode_map(&mp->scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, scales, sdims, sstr, sbox, false)) != FLINT_OK)
      return rc;
  } else {
    const uint16_t* w = static_cast<const uint16_t*>(wts->packed) + (gateup ? 0 : 2 * static_cast<size_t>(s.I) * s.d);
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows), ne};
    const cuuint64_t str[2] = {static_cast<cuuint64_t>(K) * 2, 3ull * s.I * s.d * 2};
    const cuuint32_t box[3] = {64, 128, 1};
    if ((rc = encode_map(&mp->codes, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, w, dims, str, box, true)) != FLINT_OK)
      return rc;
    mp->scales = mp->codes;
  }
  const cuuint64_t bdims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(P)};
  const cuuint64_t bstr[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t bbox[2] = {64, 64};  // one copy per 64 rows: a thread issues a copy in ~0.25 us
  return encode_map(&mp->brows, s.wd == FLINT_W_NVFP4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                    2, brows, bdims, bstr, bbox, true);
}

// Tensor maps of the tensor-core variant of the layer kernel over the gate/up
// rows of every expert: codes [E+S][2*inter][d/2] bytes, box 128 x 16 with the
// 128-byte swizzle; block scales [E+S][2*inter][d/16] bytes, box 32 x 16.
int fused_maps(FusedMaps* m, const Dims& s, const flint_moe_weights* wts) {
  const cuuint64_t ne = static_cast<cuuint64_t>(s.E + s.S);
  const cuuint64_t cdims[3] = {static_cast<cuuint64_t>(s.d / 2), static_cast<cuuint64_t>(2 * s.I), ne};
  const cuuint64_t cstr[2] = {static_cast<cuuint64_t>(s.d / 2), 3ull * s.I * s.d / 2};
  const cuuint32_t cbox[3] = {128, 16, 1};
  int rc = encode_map(&m->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, wts->packed, cdims, cstr, cbox, true);
  if (rc != FLINT_OK) return rc;
  const cuuint64_t sdims[3] = {static_cast<cuuint64_t>(s.d / 16), static_cast<cuuint64_t>(2 * s.I), ne};
  const cuuint64_t sstr[2] = {static_cast<cuuint64_t>(s.d / 16), 3ull * s.I * s.d / 16};
  const cuuint32_t sbox[3] = {32, 16, 1};
  return encode_map(&m->scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, wts->block_scales, sdims, sstr, sbox, false);
}

// Tensor maps of the batch-2..8 cluster kernel: gate/up codes [E+S][2*inter]
// [d/2] bytes (box 128 x 16, 128-byte swizzle) and block scales [E+S][2*inter]
// [d/16] (box 16 x 16); the down rows likewise from inter*d/2 code bytes and
// inter*d/16 scale bytes past each expert's base: codes [E+S][d][inter/2],
// scales [E+S][d][inter/16].
int tokn_maps(TokNMaps* m, const Dims& s, const flint_moe_weights* wts) {
  const cuuint64_t ne = static_cast<cuuint64_t>(s.E + s.S);
  const cuuint64_t cexp = 3ull * s.I * s.d / 2, sexp = 3ull * s.I * s.d / 16;
  const cuuint32_t cbox[3] = {128, 16, 1}, sbox[3] = {16, 16, 1};
  const uint8_t* codes = static_cast<const uint8_t*>(wts->packed);
  const uint8_t* scales = wts->block_scales;
  {
    const cuuint64_t cdims[3] = {static_cast<cuuint64_t>(s.d / 2), static_cast<cuuint64_t>(2 * s.I), ne};
    const cuuint64_t cstr[2] = {static_cast<cuuint64_t>(s.d / 2), cexp};
    int rc = encode_map(&m->gu_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, codes, cdims, cstr, cbox, true);
    if (rc != FLINT_OK) return rc;
    const cuuint64_t sdims[3] = {static_cast<cuuint64_t>(s.d / 16), static_cast<cuuint64_t>(2 * s.I), ne};
    const cuuint64_t sstr[2] = {static_cast<cuuint64_t>(s.d / 16), sexp};
    rc = encode_map(&m->gu_scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, scales, sdims, sstr, sbox, false);
    if (rc != FLINT_OK) return rc;
  }
  const cuuint64_t cdims[3] = {static_cast<cuuint64_t>(s.I / 2), static_cast<cuuint64_t>(s.d), ne};
  const cuuint64_t cstr[2] = {static_cast<cuuint64_t>(s.I / 2), cexp};
  int rc = encode_map(&m->dn_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, codes + static_cast<size_t>(s.I) * s.d, cdims,
                      cstr, cbox, true);
  if (rc != FLINT_OK) return rc;
  const cuuint64_t sdims[3] = {static_cast<cuuint64_t>(s.I / 16), static_cast<cuuint64_t>(s.d), ne};
  const cuuint64_t sstr[2] = {static_cast<cuuint64_t>(s.I / 16), sexp};
  return encode_map(&m->dn_scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, scales + static_cast<size_t>(s.I) * s.d / 8,
                    sdims, sstr, sbox, false);
}

// Ring depths of the tensor-core kernels for a call of T tokens: a B stage
// holds the largest expert's rows (T rounded up to whole 64-row boxes), and
// items with at most 64 tokens get two accumulators (and two MMA issuers).
// Returns the dynamic shared-memory bytes.
size_t mma_configure(MmaParams& m, int T) {
  constexpr size_t kBudget = 220 * 1024 - 1024;
  const int npad = std::min(kMmaMaxTokens, (T + 15) & ~15);
  m.b_bytes = ((npad + 63) & ~63) * 2 * kMmaSliceK;  // whole 64-row boxes, one slice of K
  m.ksplit = (npad <= kMmaMaxTokens / 2) ? 2 : 1;
  // A and B rings have the same depth (one stage of each per 128-wide K
  // slice, freed together). A stages are recycled only after their MMAs
  // complete, so the rings must cover that round trip: NVFP4 keeps 4 A stages
  // in tensor memory (columns 256..511, 64 each) fed by raw stages in the
  // shared memory left after 4 activation-row stages; bf16 weights take as
  // many A + B stage pairs as fit
  size_t wbytes, bbytes;
  if (m.nvfp4) {
    m.n_a = m.n_b = 4;
    bbytes = static_cast<size_t>(m.n_b) * m.b_bytes;
    m.n_raw = static_cast<int>(std::min<size_t>(8, (kBudget - bbytes) / kMmaRawBytes));
    wbytes = static_cast<size_t>(m.n_raw) * kMmaRawBytes;
  } else {
    m.n_raw = 1;
    m.n_a = m.n_b = static_cast<int>(std::min<size_t>(kMmaMaxStages, kBudget / (kMmaABytes + m.b_bytes)));
    bbytes = static_cast<size_t>(m.n_b) * m.b_bytes;
    wbytes = static_cast<size_t>(m.n_a) * kMmaABytes;
  }
  return 1024 + wbytes + bbytes;
}

// The tensor-core layer: router, top-k, grouping, B rows, gate/up, h rows,
// down, combine.
// ids_in / gates_in (both or neither): routing supplied by the caller, the
// router and top-k are skipped and the grouping reads these arrays.
int run_mma_path(LayerParams& p, const Dims& s, const WsLayout& w, uint8_t* ws, const flint_moe_weights* wts,
                 cudaEvent_t* ev, bool pdl, cudaStream_t st, const int32_t* ids_in = nullptr,
                 const float* gates_in = nullptr) {
  const int T = p.T, P = T * (s.k + s.S);
  MmaParams m{};
  m.x = p.x;
  m.tscale = (s.wd == FLINT_W_NVFP4) ? wts->tensor_scales : nullptr;
  m.residual = p.residual;
  m.out = p.out;
  m.status = p.status;
  m.ids = ids_in ? ids_in : p.ids;
  m.gates = ids_in ? gates_in : p.gates;
  m.ids_out = p.ids_out;
  m.gates_out = p.gates_out;
  m.rt.n_active = reinterpret_cast<int*>(ws + w.mma_n);
  m.rt.act = reinterpret_cast<int*>(ws + w.mma_act);
  m.rt.off = reinterpret_cast<int*>(ws + w.mma_off);
  m.rt.pair = reinterpret_cast<int*>(ws + w.mma_pair);
  m.rt.n_tiles = reinterpret_cast<int*>(ws + w.mma_tiles);
  const size_t max_tiles = mma_max_tiles(s, T);
  m.rt.tile_a = m.rt.n_tiles + 1;
  m.rt.tile_off = m.rt.tile_a + max_tiles;
  m.rt.tile_n = m.rt.tile_off + max_tiles;
  m.rt.mask = reinterpret_cast<uint32_t*>(ws + w.mma_mask);
  m.rt.wpre = reinterpret_cast<int*>(ws + w.mma_wpre);
  m.rt.cnt = reinterpret_cast<int*>(ws + w.mma_cnt);
  m.xrows = reinterpret_cast<uint16_t*>(ws + w.xrows);
  m.xinv = reinterpret_cast<float*>(ws + w.xinv);
  m.h = p.h;
  m.hrows = reinterpret_cast<uint16_t*>(ws + w.hrows);
  m.hinv = reinterpret_cast<float*>(ws + w.hinv);
  m.y = reinterpret_cast<float*>(ws + w.y);
  m.T = T;
  m.d = s.d;
  m.I = s.I;
  m.E = s.E;
  m.k = s.k;
  m.S = s.S;
  m.nvfp4 = (s.wd == FLINT_W_NVFP4) ? 1 : 0;
  MmaMaps gu{}, dn{};
  int rc = mma_maps(&gu, s, wts, true, m.xrows, P);
  if (rc != FLINT_OK) return rc;
  rc = mma_maps(&dn, s, wts, false, m.hrows, P);
  if (rc != FLINT_OK) return rc;

  cudaError_t e;
  if (ids_in == nullptr) {
    if (T > kMmaGroupSmallT) {  // many tokens: the router on tensor cores
      e = launch(k_router_tc, dim3((T + kRtTile - 1) / kRtTile, (s.E + kRtTile - 1) / kRtTile), dim3(256), 0, st,
                 false, p);
      if (e != cudaSuccess) return cuda_fail(e, "k_router_tc launch");
    } else {
      e = launch_router_only(p, st);
      if (e != cudaSuccess) return cuda_fail(e, "k_router_only launch");
    }
    e = launch(k_topk, dim3((T + 7) / 8), dim3(256), 0, st, pdl, p);
    if (e != cudaSuccess) return cuda_fail(e, "k_topk launch");
  }
  if (T <= kMmaGroupSmallT) {
    e = launch(k_mma_group, dim3(1), dim3(512), 0, st, pdl, m);
    if (e != cudaSuccess) return cuda_fail(e, "k_mma_group launch");
  } else {
    // prefill-size call: counting-sort grouping (mma_path.cuh)
    const int g = std::max(1, std::min(4 * num_sms(), (T * s.k + 255) / 256));
    e = launch(k_grp_zero, dim3(num_sms()), dim3(256), 0, st, pdl, m);
    if (e == cudaSuccess) e = launch(k_grp_mask, dim3(g), dim3(256), 0, st, pdl, m);
    if (e == cudaSuccess) e = launch(k_grp_scan, dim3((s.E + 7) / 8), dim3(256), 0, st, pdl, m);
    if (e == cudaSuccess) e = launch(k_grp_final, dim3(1), dim3(1024), 0, st, pdl, m);
    if (e == cudaSuccess) e = launch(k_grp_scatter, dim3(g), dim3(256), 0, st, pdl, m);
    if (e != cudaSuccess) return cuda_fail(e, "grouping launch");
  }
  e = launch(k_mma_prep, dim3((P + 7) / 8), dim3(256), 0, st, pdl, m);
  if (e != cudaSuccess) return cuda_fail(e, "k_mma_prep launch");
  const size_t smem = mma_configure(m, T);
  // tensor memory: two accumulators, plus the A stages for NVFP4 weights
  const int ncols = m.nvfp4 ? 512 : 2 * kMmaMaxTokens;
  const dim3 grid(num_sms()), block(kMmaWarps * 32);
  e = ensure_smem(reinterpret_cast<const void*>(k_mma_ffn<kEpiGateUp>));
  if (e == cudaSuccess) e = ensure_smem(reinterpret_cast<const void*>(k_mma_ffn<kEpiDown>));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  if (ev) {
    e = cudaEventRecord(ev[0], st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  }
  e = launch(k_mma_ffn<kEpiGateUp>, grid, block, smem, st, pdl && !ev, m, gu, ncols);
  if (e != cudaSuccess) return cuda_fail(e, "k_mma_ffn (gate/up) launch");
  if (ev) {
    e = cudaEventRecord(ev[1], st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  }
  e = launch(k_mma_hconv, dim3((P + 7) / 8), dim3(256), 0, st, pdl && !ev, m);
  if (e != cudaSuccess) return cuda_fail(e, "k_mma_hconv launch");
  e = launch(k_mma_ffn<kEpiDown>, grid, block, smem, st, pdl, m, dn, ncols);
  if (e != cudaSuccess) return cuda_fail(e, "k_mma_ffn (down) launch");
  e = launch(k_mma_combine, dim3((T * (s.d / 8) + 255) / 256), dim3(256), 0, st, pdl, m);
  if (e != cudaSuccess) return cuda_fail(e, "k_mma_combine launch");
  return FLINT_OK;
}

}  // namespace

// Raises a kernel's dynamic shared-memory limit on the current device, once per
// (kernel, device): for the kernels of the other translation units.
cudaError_t flint_ensure_smem(const void* kern) { return ensure_smem(kern); }
}  // namespace flint

using namespace flint;

// ======================================================================= C ABI
extern "C" {

const char* flint_last_error(void) { return g_last_error.c_str(); }

const char* flint_version(void) { return "flint_moe 0.1 (sm_100a)"; }

size_t flint_packed_bytes(const flint_moe_shape* shape) {
  Dims s;
  if (check_shape(shape, &s) != FLINT_OK) return 0;
  const size_t n = static_cast<size_t>(s.E + s.S) * 3 * s.I * s.d;
  return s.wd == FLINT_W_BF16 ? n * 2 : n / 2;
}

size_t flint_block_scale_bytes(const flint_moe_shape* shape) {
  Dims s;
  if (check_shape(shape, &s) != FLINT_OK || s.wd == FLINT_W_BF16) return 0;
  return static_cast<size_t>(s.E + s.S) * 3 * s.I * s.d / 16;
}

size_t flint_tensor_scale_bytes(const flint_moe_shape* shape) {
  Dims s;
  if (check_shape(shape, &s) != FLINT_OK || s.wd == FLINT_W_BF16) return 0;
  return static_cast<size_t>(s.E + s.S) * 3 * sizeof(float);
}

size_t flint_moe_workspace_bytes(const flint_moe_shape* shape, int32_t max_tokens) {
  Dims s;
  if (check_shape(shape, &s) != FLINT_OK || max_tokens < 0) return 0;
  return ws_layout(s, max_tokens < 1 ? 1 : max_tokens, true).total;
}

int flint_pack_nvfp4(const void* w, int32_t w_is_bf16, const flint_moe_shape* shape, void* packed,
                     uint8_t* block_scales, float* tensor_scales, void* workspace, size_t ws_bytes,
                     void* stream) {
  Dims s;
  int rc = check_shape(shape, &s);
  if (rc != FLINT_OK) return rc;
  if (s.wd != FLINT_W_NVFP4) return fail(FLINT_ERR_INVALID_ARG, "flint_pack_nvfp4 needs wdtype FLINT_W_NVFP4");
  if (!w || !packed || !block_scales || !tensor_scales || !workspace)
    return fail(FLINT_ERR_INVALID_ARG, "flint_pack_nvfp4: NULL pointer");
  if (!aligned16(w) || !aligned16(packed) || !aligned16(block_scales) || !aligned16(tensor_scales) ||
      !aligned16(workspace))
    return fail(FLINT_ERR_MISALIGNED, "flint_pack_nvfp4: pointers must be 16-byte aligned");
  const WsLayout lay = ws_layout(s, 1, false);
  if (ws_bytes < lay.total) return fail(FLINT_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, lay.total);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int n_mats = (s.E + s.S) * 3;
  const long long per_mat = static_cast<long long>(s.I) * s.d;
  unsigned* amax = reinterpret_cast<unsigned*>(ws + lay.amax);
  int* status = reinterpret_cast<int*>(ws + lay.status);
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(unsigned) * n_mats, st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  const dim3 ga(32, n_mats);
  if (w_is_bf16)
    k_pack_amax<true><<<ga, 256, 0, st>>>(w, per_mat, amax, status);
  else
    k_pack_amax<false><<<ga, 256, 0, st>>>(w, per_mat, amax, status);
  const long long n_blocks = static_cast<long long>(n_mats) * per_mat / 16;
  const unsigned gq = static_cast<unsigned>((n_blocks + 255) / 256);
  const long long cpe = 3LL * s.I * s.d / 2, spe = 3LL * s.I * s.d / 16;
  if (w_is_bf16)
    k_pack_quant<true><<<gq, 256, 0, st>>>(w, s.d, s.I, n_blocks, cpe, spe, amax,
                                           static_cast<uint8_t*>(packed), block_scales, tensor_scales);
  else
    k_pack_quant<false><<<gq, 256, 0, st>>>(w, s.d, s.I, n_blocks, cpe, spe, amax,
                                            static_cast<uint8_t*>(packed), block_scales, tensor_scales);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "flint_pack_nvfp4 launch");
  return FLINT_OK;
}

int flint_pack_bf16(const uint16_t* w, const flint_moe_shape* shape, uint16_t* packed, void* stream) {
  Dims s;
  int rc = check_shape(shape, &s);
  if (rc != FLINT_OK) return rc;
  if (s.wd != FLINT_W_BF16) return fail(FLINT_ERR_INVALID_ARG, "flint_pack_bf16 needs wdtype FLINT_W_BF16");
  if (!w || !packed) return fail(FLINT_ERR_INVALID_ARG, "flint_pack_bf16: NULL pointer");
  if (!aligned16(w) || !aligned16(packed)) return fail(FLINT_ERR_MISALIGNED, "flint_pack_bf16: unaligned pointer");
  const long long n_vec = static_cast<long long>(s.E + s.S) * 3 * s.I * s.d / 8;
  k_pack_bf16<<<static_cast<unsigned>((n_vec + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      w, s.d, s.I, n_vec, packed);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "flint_pack_bf16 launch");
  return FLINT_OK;
}

int flint_pack_nvfp4_dense(const void* w, int32_t w_is_bf16, int32_t rows, int32_t cols, uint8_t* codes,
                           uint8_t* scales, float* tensor_scale, void* workspace, size_t ws_bytes, void* stream) {
  if (!w || !codes || !scales || !tensor_scale || !workspace)
    return fail(FLINT_ERR_INVALID_ARG, "flint_pack_nvfp4_dense: NULL pointer");
  if (rows < 1 || !(cols == 512 || cols == 1024 || cols == 2048 || cols == 4096))
    return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "flint_pack_nvfp4_dense: rows=%d cols=%d (cols one of 512..4096)", rows, cols);
  if (!aligned16(w) || !aligned16(codes) || !aligned16(scales) || !aligned16(tensor_scale) || !aligned16(workspace))
    return fail(FLINT_ERR_MISALIGNED, "flint_pack_nvfp4_dense: pointers must be 16-byte aligned");
  if (ws_bytes < kCtrlBytes + 256) return fail(FLINT_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, kCtrlBytes + 256);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  unsigned* amax = reinterpret_cast<unsigned*>(ws + kCtrlBytes);
  int* status = reinterpret_cast<int*>(ws);
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(unsigned), st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  const long long n = static_cast<long long>(rows) * cols;
  if (w_is_bf16)
    k_pack_amax<true><<<dim3(1024, 1), 256, 0, st>>>(w, n, amax, status);
  else
    k_pack_amax<false><<<dim3(1024, 1), 256, 0, st>>>(w, n, amax, status);
  const long long n_blocks = n / 16;
  const unsigned g = static_cast<unsigned>((n_blocks + 255) / 256);
  if (w_is_bf16)
    k_pack_dense_quant<true><<<g, 256, 0, st>>>(w, rows, cols, amax, codes, scales, tensor_scale);
  else
    k_pack_dense_quant<false><<<g, 256, 0, st>>>(w, rows, cols, amax, codes, scales, tensor_scale);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "flint_pack_nvfp4_dense launch");
  return FLINT_OK;
}

int flint_lm_head(const uint16_t* x, int32_t T, const uint8_t* codes, const uint8_t* scales,
                  const float* tensor_scale, int32_t rows, int32_t cols, float* out, void* workspace,
                  size_t ws_bytes, void* stream) {
  if (!x || !codes || !scales || !tensor_scale || !out || !workspace)
    return fail(FLINT_ERR_INVALID_ARG, "flint_lm_head: NULL pointer");
  if (T < 0) return fail(FLINT_ERR_INVALID_ARG, "T=%d", T);
  if (T == 0) return FLINT_OK;
  if (rows < 1 || !(cols == 512 || cols == 1024 || cols == 2048 || cols == 4096))
    return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "flint_lm_head: rows=%d cols=%d (cols one of 512..4096)", rows, cols);
  if (T > kLmMaxTokens) return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "flint_lm_head: at most %d tokens", kLmMaxTokens);
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(tensor_scale) || !aligned16(out) ||
      !aligned16(workspace))
    return fail(FLINT_ERR_MISALIGNED, "flint_lm_head: pointers must be 16-byte aligned");
  if (ws_bytes < 4) return fail(FLINT_ERR_WORKSPACE, "workspace %zu < 4 bytes", ws_bytes);
  LmHeadParams p{};
  p.x = x;
  p.tscale = tensor_scale;
  p.out = out;
  p.status = static_cast<int*>(workspace);
  p.T = T;
  p.V = rows;
  LmMaps maps;
  const cuuint64_t cdims[2] = {static_cast<cuuint64_t>(cols / 2), static_cast<cuuint64_t>(rows)};
  const cuuint64_t cstr[1] = {static_cast<cuuint64_t>(cols / 2)};
  const cuuint32_t cbox[2] = {128, 16};
  int rc = encode_map(&maps.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, codes, cdims, cstr, cbox, true);
  if (rc != FLINT_OK) return rc;
  const cuuint64_t sdims[2] = {static_cast<cuuint64_t>(cols / 16), static_cast<cuuint64_t>(rows)};
  const cuuint64_t sstr[1] = {static_cast<cuuint64_t>(cols / 16)};
  const cuuint32_t sbox[2] = {32, 16};
  rc = encode_map(&maps.scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, scales, sdims, sstr, sbox, false);
  if (rc != FLINT_OK) return rc;
  cudaError_t e = lm_head_launch(cols, p, maps, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "k_lm_head launch");
  return FLINT_OK;
}

int flint_moe_route(const uint16_t* x, int32_t T, const uint16_t* router_w, const flint_moe_shape* shape,
                    int32_t* topk_ids, float* topk_weights, void* workspace, size_t ws_bytes, void* stream) {
  Dims s;
  int rc = check_shape(shape, &s);
  if (rc != FLINT_OK) return rc;
  if (T < 0) return fail(FLINT_ERR_INVALID_ARG, "T=%d", T);
  if (T == 0) return FLINT_OK;
  if (!x || !router_w || !topk_ids || !topk_weights || !workspace)
    return fail(FLINT_ERR_INVALID_ARG, "flint_moe_route: NULL pointer");
  if (!aligned16(x) || !aligned16(router_w) || !aligned16(topk_ids) || !aligned16(topk_weights) ||
      !aligned16(workspace))
    return fail(FLINT_ERR_MISALIGNED, "flint_moe_route: pointers must be 16-byte aligned");
  const WsLayout lay = ws_layout(s, T, false);
  if (ws_bytes < lay.total) return fail(FLINT_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, lay.total);
  LayerParams p{};
  fill_common(p, s, lay, static_cast<uint8_t*>(workspace), T);
  p.x = x;
  p.wr = router_w;
  p.ids = topk_ids;
  p.gates = topk_weights;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (T > kMmaGroupSmallT) {  // many tokens: the router on tensor cores
    e = launch(k_router_tc, dim3((T + kRtTile - 1) / kRtTile, (s.E + kRtTile - 1) / kRtTile), dim3(256), 0, st,
               false, p);
    if (e != cudaSuccess) return cuda_fail(e, "k_router_tc launch");
  } else {
    e = launch_router_only(p, st);
    if (e != cudaSuccess) return cuda_fail(e, "k_router_only launch");
  }
  e = launch(k_topk, dim3((T + 7) / 8), dim3(256), 0, st, true, p);
  if (e != cudaSuccess) return cuda_fail(e, "k_topk launch");
  return FLINT_OK;
}

int flint_moe_forward_ex(const uint16_t* x, int32_t T, const uint16_t* router_w,
                         const flint_moe_weights* weights, const flint_moe_shape* shape,
                         const uint16_t* residual, uint16_t* out, void* workspace, size_t ws_bytes,
                         const flint_moe_options* options, void* stream) {
  Dims s;
  int rc = check_shape(shape, &s);
  if (rc != FLINT_OK) return rc;
  if (T < 0) return fail(FLINT_ERR_INVALID_ARG, "T=%d", T);
  if (T == 0) return FLINT_OK;
  if (!x || !router_w || !weights || !weights->packed || !out || !workspace)
    return fail(FLINT_ERR_INVALID_ARG, "flint_moe_forward: NULL pointer");
  if (s.wd == FLINT_W_NVFP4 && (!weights->block_scales || !weights->tensor_scales))
    return fail(FLINT_ERR_INVALID_ARG, "flint_moe_forward: NVFP4 weights need block and tensor scales");
  if (!aligned16(x) || !aligned16(router_w) || !aligned16(weights->packed) || !aligned16(out) ||
      !aligned16(workspace) || (residual && !aligned16(residual)) ||
      (weights->block_scales && !aligned16(weights->block_scales)) ||
      (weights->tensor_scales && !aligned16(weights->tensor_scales)))
    return fail(FLINT_ERR_MISALIGNED, "flint_moe_forward: pointers must be 16-byte aligned");
  const int path = options ? options->path : FLINT_PATH_AUTO;
  const bool pdl = options ? options->use_pdl != 0 : true;
  if (path < FLINT_PATH_AUTO || path > FLINT_PATH_MMA) return fail(FLINT_ERR_INVALID_ARG, "path %d", path);
  if (options && ((options->topk_ids == nullptr) != (options->topk_weights == nullptr)))
    return fail(FLINT_ERR_INVALID_ARG, "topk_ids and topk_weights go together");
  const int variant = options ? options->layer_variant : FLINT_LAYER_AUTO;
  if (variant < FLINT_LAYER_AUTO || variant > FLINT_LAYER_CLUSTER)
    return fail(FLINT_ERR_INVALID_ARG, "layer_variant %d", variant);
  if (variant == FLINT_LAYER_CLUSTER && (T > kTnMaxTokens || path == FLINT_PATH_MMA || s.wd != FLINT_W_NVFP4))
    return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "the cluster kernels take 1..%d tokens and NVFP4 weights (T=%d)",
                kTnMaxTokens, T);
  const bool use_gemv = (path == FLINT_PATH_GEMV) ||
                        (path == FLINT_PATH_AUTO && T < kMaxGemvTokens && s.wd == FLINT_W_NVFP4);
  if (use_gemv) {
    if (s.wd != FLINT_W_NVFP4)
      return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "the GEMV path takes NVFP4 weights; bf16 weights use the tensor-core path");
    const int gemv_max_t = (s.d == 4096) ? kMaxGemvTokens / 2 : kMaxGemvTokens;
    if (T > gemv_max_t)
      return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "GEMV path takes at most %d tokens at d=%d", gemv_max_t, s.d);
  } else {
    if (T > kMmaMaxCallTokens)
      return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "tensor-core path takes at most %d tokens (T=%d)", kMmaMaxCallTokens, T);
    if (T > kMmaGroupSmallT && s.E + s.S > 1024)
      return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "more than %d tokens need E + S <= 1024", kMmaGroupSmallT);
    if (s.wd == FLINT_W_NVFP4 && s.I < 256)
      return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "tensor-core path with NVFP4 weights needs inter >= 256 (inter=%d)", s.I);
    if (options && options->input_rmsnorm)
      return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "input_rmsnorm is a GEMV-path option");
  }
  const WsLayout lay = ws_layout(s, T, !use_gemv);
  if (ws_bytes < lay.total) return fail(FLINT_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, lay.total);

  LayerParams p{};
  fill_common(p, s, lay, static_cast<uint8_t*>(workspace), T);
  p.x = x;
  p.wr = router_w;
  p.codes = static_cast<const uint8_t*>(weights->packed);
  p.scales = weights->block_scales;
  p.tscale = weights->tensor_scales;
  p.residual = residual;
  p.out = out;
  if (options && options->topk_ids) {
    p.ids_out = options->topk_ids;
    p.gates_out = options->topk_weights;
  }
  p.input_norm = (options && options->input_rmsnorm) ? 1 : 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaEvent_t* ev = options ? static_cast<cudaEvent_t*>(options->profile_events) : nullptr;
  if (!use_gemv) return run_mma_path(p, s, lay, static_cast<uint8_t*>(workspace), weights, ev, pdl, st);
  const bool split = options && options->split_kernels;
  if (T == 1 && !split && (variant == FLINT_LAYER_AUTO || variant == FLINT_LAYER_CLUSTER)) {
    // one token: one cluster of CTAs per selected expert and one for the shared
    // expert (tok1.cuh), when the shape fits it on this device
    Tok1Params t{};
    t.x = x;
    t.wr = router_w;
    t.codes = p.codes;
    t.scales = p.scales;
    t.tscale = p.tscale;
    t.residual = residual;
    t.out = out;
    t.status = p.status;
    t.rb_count = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(workspace) + lay.rb_count);
    t.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + lay.tok1_part);
    t.ids = p.ids;
    t.gates = p.gates;
    t.ids_out = p.ids_out;
    t.gates_out = p.gates_out;
    t.cpe = p.cpe;
    t.spe = p.spe;
    t.E = s.E;
    t.k = s.k;
    t.S = s.S;
    t.input_norm = p.input_norm;
    t.trigger_early = 1;
    if (tok1_dispatch(s.d, s.I, s.E, false, &t, pdl, st, nullptr)) {
      if (ev) {
        cudaError_t e = cudaEventRecord(ev[0], st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
      }
      cudaError_t e = cudaSuccess;
      tok1_dispatch(s.d, s.I, s.E, true, &t, pdl && !ev, st, &e);
      if (e != cudaSuccess) return cuda_fail(e, "k_tok1 launch");
      if (ev) {
        e = cudaEventRecord(ev[1], st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
      }
      return FLINT_OK;
    }
    if (variant == FLINT_LAYER_CLUSTER)
      return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "the cluster kernel does not fit this shape on this device");
  }
  if (T >= 2 && T <= kTnMaxTokens && !split && variant == FLINT_LAYER_CLUSTER) {
    // 2..8 tokens, on request: persistent 16-CTA clusters taking the selected
    // experts in turn (tokn.cuh), when the shape fits it on this device (AUTO
    // keeps the persistent layer kernel, measured faster at these batches)
    TokNParams t{};
    t.x = x;
    t.wr = router_w;
    t.codes = p.codes;
    t.scales = p.scales;
    t.cpe = p.cpe;
    t.spe = p.spe;
    t.tscale = p.tscale;
    t.residual = residual;
    t.out = out;
    t.status = p.status;
    t.rb_count = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(workspace) + lay.rb_count);
    t.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + lay.tok1_part);
    t.ids = p.ids;
    t.gates = p.gates;
    t.ids_out = p.ids_out;
    t.gates_out = p.gates_out;
    t.T = T;
    t.E = s.E;
    t.k = s.k;
    t.S = s.S;
    t.input_norm = p.input_norm;
    if (tokn_dispatch(s.d, s.I, s.E, T, false, &t, nullptr, pdl, st, nullptr)) {
      TokNMaps maps;
      const int rc = tokn_maps(&maps, s, weights);
      if (rc != FLINT_OK) return rc;
      if (ev) {
        cudaError_t e = cudaEventRecord(ev[0], st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
      }
      cudaError_t e = cudaSuccess;
      tokn_dispatch(s.d, s.I, s.E, T, true, &t, &maps, pdl && !ev, st, &e);
      if (e != cudaSuccess) return cuda_fail(e, "k_tokn launch");
      if (ev) {
        e = cudaEventRecord(ev[1], st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
      }
      return FLINT_OK;
    }
    if (variant == FLINT_LAYER_CLUSTER)
      return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "the cluster kernel does not fit this shape on this device");
  }
  if (T <= kFusedMaxTokens && !split) {
    bool tc = variant == FLINT_LAYER_MMA || (variant == FLINT_LAYER_AUTO && T >= kTcMinTokens);
    size_t smem = configure_fused(p, s, T, tc);
    if (smem == 0 && tc && variant == FLINT_LAYER_AUTO) {
      tc = false;
      smem = configure_fused(p, s, T, false);
    }
    FusedMaps maps;
    if (smem > 0 && tc) {
      const int rc = fused_maps(&maps, s, weights);
      if (rc != FLINT_OK) return rc;
    }
    if (smem > 0) {
      if (ev) {
        cudaError_t e = cudaEventRecord(ev[0], st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
      }
      cudaError_t e = launch_fused(p, tc ? &maps : nullptr, smem, st);
      if (e != cudaSuccess) return cuda_fail(e, "k_layer launch");
      if (ev) {
        e = cudaEventRecord(ev[1], st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
      }
      return FLINT_OK;
    }
  }
  configure(p, s, T);
  cudaError_t e = launch_route_fwd(p, st, pdl);
  if (e != cudaSuccess) return cuda_fail(e, "k_route launch");
  if (ev) {
    e = cudaEventRecord(ev[0], st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  }
  e = launch_gateup(p, st, pdl && !ev);
  if (e != cudaSuccess) return cuda_fail(e, "k_gateup launch");
  if (ev) {
    e = cudaEventRecord(ev[1], st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  }
  e = launch_down(p, st, pdl && !ev);
  if (e != cudaSuccess) return cuda_fail(e, "k_down launch");
  return FLINT_OK;
}

int flint_moe_forward(const uint16_t* x, int32_t T, const uint16_t* router_w, const flint_moe_weights* weights,
                      const flint_moe_shape* shape, const uint16_t* residual, uint16_t* out, void* workspace,
                      size_t ws_bytes, void* stream) {
  return flint_moe_forward_ex(x, T, router_w, weights, shape, residual, out, workspace, ws_bytes, nullptr,
                              stream);
}

int flint_moe_forward_routed(const uint16_t* x, int32_t T, const int32_t* topk_ids, const float* topk_weights,
                             const flint_moe_weights* weights, const flint_moe_shape* shape,
                             const uint16_t* residual, uint16_t* out, void* workspace, size_t ws_bytes,
                             void* stream) {
  Dims s;
  int rc = check_shape(shape, &s);
  if (rc != FLINT_OK) return rc;
  if (T < 0) return fail(FLINT_ERR_INVALID_ARG, "T=%d", T);
  if (T == 0) return FLINT_OK;
  if (!x || !topk_ids || !topk_weights || !weights || !weights->packed || !out || !workspace)
    return fail(FLINT_ERR_INVALID_ARG, "flint_moe_forward_routed: NULL pointer");
  if (s.wd == FLINT_W_NVFP4 && (!weights->block_scales || !weights->tensor_scales))
    return fail(FLINT_ERR_INVALID_ARG, "flint_moe_forward_routed: NVFP4 weights need block and tensor scales");
  if (!aligned16(x) || !aligned16(weights->packed) || !aligned16(out) || !aligned16(workspace) ||
      (residual && !aligned16(residual)) || (weights->block_scales && !aligned16(weights->block_scales)) ||
      (weights->tensor_scales && !aligned16(weights->tensor_scales)) ||
      (reinterpret_cast<uintptr_t>(topk_ids) & 3u) || (reinterpret_cast<uintptr_t>(topk_weights) & 3u))
    return fail(FLINT_ERR_MISALIGNED, "flint_moe_forward_routed: misaligned pointer");
  if (T > kMmaMaxCallTokens)
    return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "tensor-core path takes at most %d tokens (T=%d)", kMmaMaxCallTokens, T);
  if (T > kMmaGroupSmallT && s.E + s.S > 1024)
    return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "more than %d tokens need E + S <= 1024", kMmaGroupSmallT);
  if (s.wd == FLINT_W_NVFP4 && s.I < 256)
    return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "tensor-core path with NVFP4 weights needs inter >= 256 (inter=%d)", s.I);
  const WsLayout lay = ws_layout(s, T, true);
  if (ws_bytes < lay.total) return fail(FLINT_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, lay.total);
  LayerParams p{};
  fill_common(p, s, lay, static_cast<uint8_t*>(workspace), T);
  p.x = x;
  p.codes = static_cast<const uint8_t*>(weights->packed);
  p.scales = weights->block_scales;
  p.tscale = weights->tensor_scales;
  p.residual = residual;
  p.out = out;
  return run_mma_path(p, s, lay, static_cast<uint8_t*>(workspace), weights, nullptr, true,
                      static_cast<cudaStream_t>(stream), topk_ids, topk_weights);
}

int flint_moe_workspace_init(void* workspace, size_t ws_bytes, void* stream) {
  if (!workspace) return fail(FLINT_ERR_INVALID_ARG, "workspace is NULL");
  if (!aligned16(workspace)) return fail(FLINT_ERR_MISALIGNED, "workspace must be 16-byte aligned");
  if (ws_bytes < kCtrlBytes) return fail(FLINT_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, kCtrlBytes);
  cudaError_t e = cudaMemsetAsync(workspace, 0, ws_bytes, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  return FLINT_OK;
}

int flint_moe_get_status(void* workspace, int32_t* device_flags, void* stream) {
  if (!workspace) return fail(FLINT_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t flags = 0;
  cudaError_t e = cudaMemcpyAsync(&flags, workspace, sizeof flags, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, sizeof flags, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "flint_moe_get_status");
  if (device_flags) *device_flags = flags;
  if (flags & FLINT_DEVCHECK_WAIT) return fail(FLINT_ERR_TIMEOUT, "a bounded device wait ran out");
  if (flags) return fail(FLINT_ERR_DEVICE_CHECK, "device check flags 0x%x", flags);
  return FLINT_OK;
}

int flint_debug_decode(const flint_moe_weights* weights, const flint_moe_shape* shape, int32_t expert,
                       int32_t matrix, int32_t decoder, int32_t row0, int32_t rows, int32_t k0, int32_t kn, float* out,
                       void* stream) {
  Dims s;
  int rc = check_shape(shape, &s);
  if (rc != FLINT_OK) return rc;
  if (s.wd != FLINT_W_NVFP4 || !weights || !weights->packed || !weights->block_scales || !out)
    return fail(FLINT_ERR_INVALID_ARG, "flint_debug_decode: NVFP4 weights and output needed");
  if (expert < 0 || expert >= s.E + s.S || (matrix != 0 && matrix != 1) || decoder < 0 || decoder > 1)
    return fail(FLINT_ERR_INVALID_ARG, "flint_debug_decode: bad expert/matrix/decoder");
  const int K = matrix == 0 ? s.d : s.I, nrows = matrix == 0 ? 2 * s.I : s.d;
  const int th = decoder == 0 ? 128 : 16, tw = decoder == 0 ? 256 : 128;
  if (row0 < 0 || rows <= 0 || rows % th || row0 + rows > nrows || k0 < 0 || kn <= 0 || kn % tw || k0 % tw ||
      k0 + kn > K)
    return fail(FLINT_ERR_INVALID_ARG, "flint_debug_decode: tiles of %d rows x %d K inside the matrix", th, tw);
  const long long cpe = 3LL * s.I * s.d / 2, spe = 3LL * s.I * s.d / 16;
  const uint8_t* codes = static_cast<const uint8_t*>(weights->packed) + expert * cpe +
                         (matrix == 0 ? 0 : static_cast<long long>(s.I) * s.d) + static_cast<long long>(row0) * (K / 2);
  const uint8_t* scales = weights->block_scales + expert * spe +
                          (matrix == 0 ? 0 : static_cast<long long>(s.I) * s.d / 8) + static_cast<long long>(row0) * (K / 16);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (decoder == 0)
    k_debug_decode_tmem<<<dim3(rows / 128, kn / 256), 512, 0, st>>>(codes, scales, K, k0, out, kn);
  else
    k_debug_decode_frag<<<dim3(rows / 16, kn / 128), 32, 0, st>>>(codes, scales, K, k0, out, kn);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "flint_debug_decode");
  return FLINT_OK;
}

int flint_debug_group(const int32_t* ids, int32_t T, const flint_moe_shape* shape, int32_t impl, int32_t* act,
                      int32_t* off, int32_t* pair, int32_t* counts, void* workspace, size_t ws_bytes, void* stream) {
  Dims s;
  int rc = check_shape(shape, &s);
  if (rc != FLINT_OK) return rc;
  if (!ids || !act || !off || !pair || !counts || !workspace)
    return fail(FLINT_ERR_INVALID_ARG, "flint_debug_group: NULL pointer");
  if (impl < 0 || impl > 3) return fail(FLINT_ERR_INVALID_ARG, "flint_debug_group: impl %d", impl);
  const int max_t = impl == 0 ? kMmaGroupSmallT
                              : (impl == 1 ? 64 / s.k : (impl == 2 ? kMaxGemvTokens : kMmaMaxCallTokens));
  if (T < 1 || T > max_t) return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "flint_debug_group: impl %d takes 1..%d tokens", impl, max_t);
  if (ws_bytes < kCtrlBytes) return fail(FLINT_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, kCtrlBytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (impl == 3) {
    // the tensor-core path's counting-sort grouping, scratch after the control block
    if (s.E + s.S > 1024) return fail(FLINT_ERR_UNSUPPORTED_SHAPE, "flint_debug_group: impl 3 needs E + S <= 1024");
    const size_t tiles = mma_max_tiles(s, T), words = static_cast<size_t>(s.E) * ((T + 31) / 32);
    const size_t need = kCtrlBytes + al256(sizeof(int) * (1 + 3 * tiles)) + 2 * al256(4 * words) + al256(4 * s.E);
    if (ws_bytes < need) return fail(FLINT_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
    uint8_t* w = static_cast<uint8_t*>(workspace);
    MmaParams m{};
    m.ids = ids;
    m.status = static_cast<int*>(workspace);
    m.T = T;
    m.E = s.E;
    m.k = s.k;
    m.S = s.S;
    m.rt.act = act;
    m.rt.off = off;
    m.rt.pair = pair;
    m.rt.n_active = counts + 1;
    size_t o = kCtrlBytes;
    m.rt.n_tiles = reinterpret_cast<int*>(w + o);
    m.rt.tile_a = m.rt.n_tiles + 1;
    m.rt.tile_off = m.rt.tile_a + tiles;
    m.rt.tile_n = m.rt.tile_off + tiles;
    o += al256(sizeof(int) * (1 + 3 * tiles));
    m.rt.mask = reinterpret_cast<uint32_t*>(w + o);
    o += al256(4 * words);
    m.rt.wpre = reinterpret_cast<int*>(w + o);
    o += al256(4 * words);
    m.rt.cnt = reinterpret_cast<int*>(w + o);
    const int g = std::max(1, std::min(4 * num_sms(), (T * s.k + 255) / 256));
    cudaError_t e = launch(k_grp_zero, dim3(num_sms()), dim3(256), 0, st, false, m);
    if (e == cudaSuccess) e = launch(k_grp_mask, dim3(g), dim3(256), 0, st, false, m);
    if (e == cudaSuccess) e = launch(k_grp_scan, dim3((s.E + 7) / 8), dim3(256), 0, st, false, m);
    if (e == cudaSuccess) e = launch(k_grp_final, dim3(1), dim3(1024), 0, st, false, m);
    if (e == cudaSuccess) e = launch(k_grp_scatter, dim3(g), dim3(256), 0, st, false, m);
    if (e == cudaSuccess) {
      k_debug_routed_count<<<1, 1, 0, st>>>(counts, s.S);
      e = cudaGetLastError();
    }
    if (e != cudaSuccess) return cuda_fail(e, "grouping launch");
    return FLINT_OK;
  }
  k_debug_group<<<1, 512, 0, st>>>(ids, T, s.k, s.E, s.S, impl, act, off, pair, counts, static_cast<int*>(workspace));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "k_debug_group launch");
  return FLINT_OK;
}

int flint_debug_dequant(const flint_moe_weights* weights, const flint_moe_shape* shape, int32_t expert,
                        int32_t matrix, int32_t row0, int32_t rows, float* out, float* tensor_scale_out,
                        void* stream) {
  Dims s;
  int rc = check_shape(shape, &s);
  if (rc != FLINT_OK) return rc;
  if (s.wd != FLINT_W_NVFP4 || !weights || !weights->packed || !weights->block_scales ||
      !weights->tensor_scales || !out)
    return fail(FLINT_ERR_INVALID_ARG, "flint_debug_dequant: NVFP4 weights and output needed");
  if (expert < 0 || expert >= s.E + s.S || (matrix != 0 && matrix != 1) || row0 < 0 || rows < 0)
    return fail(FLINT_ERR_INVALID_ARG, "flint_debug_dequant: bad expert/matrix/rows");
  const int max_rows = matrix == 0 ? s.I : s.d;
  if (row0 + rows > max_rows) return fail(FLINT_ERR_INVALID_ARG, "flint_debug_dequant: rows out of range");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long cpe = 3LL * s.I * s.d / 2, spe = 3LL * s.I * s.d / 16;
  const uint8_t* codes = static_cast<const uint8_t*>(weights->packed) + expert * cpe;
  const uint8_t* scales = weights->block_scales + expert * spe;
  int K;
  long long nrows;
  if (matrix == 0) {  // units: gate row, up row
    codes += static_cast<long long>(row0) * s.d;
    scales += static_cast<long long>(row0) * s.d / 8;
    K = s.d;
    nrows = 2LL * rows;
  } else {
    codes += static_cast<long long>(s.I) * s.d + static_cast<long long>(row0) * s.I / 2;
    scales += static_cast<long long>(s.I) * s.d / 8 + static_cast<long long>(row0) * s.I / 16;
    K = s.I;
    nrows = rows;
  }
  const long long nv = nrows * (K / 32);
  if (nv > 0)
    k_debug_dequant<<<static_cast<unsigned>((nv + 255) / 256), 256, 0, st>>>(codes, scales, K, nrows, out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "k_debug_dequant launch");
  if (tensor_scale_out) {
    e = cudaMemcpyAsync(tensor_scale_out, weights->tensor_scales + 3 * expert + (matrix == 0 ? 0 : 2),
                        (matrix == 0 ? 2 : 1) * sizeof(float), cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync");
  }
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  return FLINT_OK;
}

// ---------------------------------------------------------------------------
// Layer forward for callers that cannot allocate device memory: the scratch
// lives in a fixed, file-scope device array instead of a caller workspace.
// ---------------------------------------------------------------------------
}  // extern "C"

namespace flint {
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB, held by every device that loads the library
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// The scratch's device address per CUDA context, keyed by the context's
// unique id (cuCtxGetId never repeats an id within a process, so a context
// created after cudaDeviceReset, or another driver context of the same
// device, gets its own entry and its own lookup), with the shape of the last
// call that ran on it.
struct NoAllocSlot {
  unsigned long long ctx_id;
  void* addr;
  bool have_shape;
  Dims last;
};
std::mutex g_noalloc_mu;
NoAllocSlot g_noalloc_slots[64];
int g_noalloc_n = 0;

typedef CUresult (*PFN_ctx_get_current)(CUcontext*);
typedef CUresult (*PFN_ctx_get_id)(CUcontext, unsigned long long*);

int current_context_id(unsigned long long* id) {
  static PFN_ctx_get_current get_current = nullptr;
  static PFN_ctx_get_id get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_ctx_get_current>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_ctx_get_id>(f);
  });
  if (get_current == nullptr || get_id == nullptr)
    return fail(FLINT_ERR_CUDA, "cuCtxGetCurrent / cuCtxGetId are not available");
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return fail(FLINT_ERR_CUDA, "cuCtxGetCurrent failed");
  if (ctx == nullptr) {
    // nothing current yet: bind the current device's primary context, as the
    // runtime's first call on this thread would
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaSetDevice(dev);
    if (e != cudaSuccess) return cuda_fail(e, "context set-up");
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return fail(FLINT_ERR_CUDA, "no current CUDA context");
  }
  if (get_id(ctx, id) != CUDA_SUCCESS) return fail(FLINT_ERR_CUDA, "cuCtxGetId failed");
  return FLINT_OK;
}

// The slot of the current context, created (with the symbol lookup, done with
// that context current) on first use. Called with g_noalloc_mu held.
int noalloc_slot(NoAllocSlot** out) {
  unsigned long long id = 0;
  int rc = current_context_id(&id);
  if (rc != FLINT_OK) return rc;
  for (int i = 0; i < g_noalloc_n; ++i)
    if (g_noalloc_slots[i].ctx_id == id) {
      *out = &g_noalloc_slots[i];
      return FLINT_OK;
    }
  // Host code cannot use the array's name as a device address: look the
  // address up in this context.
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
  const bool evict = g_noalloc_n >= 64;
  NoAllocSlot* s = &g_noalloc_slots[evict ? (id % 64) : g_noalloc_n++];
  s->ctx_id = id;
  s->addr = p;
  // a context seen for the first time has a freshly loaded (zero) array; one
  // whose slot was evicted earlier may not, so its next call zeroes it
  s->have_shape = evict;
  s->last = Dims{0, 0, 0, 0, 0, 0};
  *out = s;
  return FLINT_OK;
}

bool same_dims(const Dims& a, const Dims& b) {
  return a.d == b.d && a.I == b.I && a.E == b.E && a.k == b.k && a.S == b.S && a.wd == b.wd;
}
}  // namespace
}  // namespace flint

extern "C" {

int flint_moe_forward_noalloc(const uint16_t* x, int32_t T, const uint16_t* router_w,
                              const flint_moe_weights* weights, const flint_moe_shape* shape,
                              const uint16_t* residual, uint16_t* out, void* stream) {
  Dims s;
  int rc = check_shape(shape, &s);
  if (rc != FLINT_OK) return rc;
  if (T < 0) return fail(FLINT_ERR_INVALID_ARG, "T=%d", T);
  if (T == 0) return FLINT_OK;
  // the path flint_moe_forward takes for this call (options == NULL: automatic)
  const bool mma = !(T < kMaxGemvTokens && s.wd == FLINT_W_NVFP4);
  const size_t need = ws_layout(s, T, mma).total;
  if (need > kNoAllocScratchBytes)
    return fail(FLINT_ERR_WORKSPACE,
                "flint_moe_forward_noalloc: this call needs %zu bytes of scratch; the built-in scratch holds %zu "
                "(use flint_moe_forward with a caller workspace)",
                need, kNoAllocScratchBytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    NoAllocSlot* slot = nullptr;
    rc = noalloc_slot(&slot);
    if (rc != FLINT_OK) return rc;
    scratch = slot->addr;
    // The persistent kernel's launch tags need the control block's generation
    // word and the tagged regions (at offsets that depend on the shape) to
    // hold only older tags. The array is zero when the module loads; after a
    // shape change, everything but the status word (byte 0, kept for
    // flint_moe_noalloc_get_status) is zeroed again. Calls of one shape keep
    // the contents: the tags of later launches are newer.
    if (slot->have_shape && !same_dims(slot->last, s)) {
      cudaError_t e = cudaMemsetAsync(static_cast<uint8_t*>(scratch) + 4, 0, kNoAllocScratchBytes - 4, st);
      if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    }
    slot->last = s;
    slot->have_shape = true;
  }
  return flint_moe_forward_ex(x, T, router_w, weights, shape, residual, out, scratch, kNoAllocScratchBytes,
                              nullptr, stream);
}

int flint_moe_noalloc_get_status(int32_t* device_flags, void* stream) {
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    NoAllocSlot* slot = nullptr;
    const int rc = noalloc_slot(&slot);
    if (rc != FLINT_OK) return rc;
    scratch = slot->addr;
  }
  return flint_moe_get_status(scratch, device_flags, stream);
}

int flint_debug_noalloc_scratch(void** addr) {
  if (!addr) return fail(FLINT_ERR_INVALID_ARG, "addr is NULL");
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  NoAllocSlot* slot = nullptr;
  const int rc = noalloc_slot(&slot);
  if (rc != FLINT_OK) return rc;
  *addr = slot->addr;
  return FLINT_OK;
}

int flint_debug_wait_timeout(void* workspace, int64_t cycles, void* stream) {
  if (!workspace) return fail(FLINT_ERR_INVALID_ARG, "workspace is NULL");
  if (!aligned16(workspace)) return fail(FLINT_ERR_MISALIGNED, "workspace must be 16-byte aligned");
  long long c = cycles < 1 ? 1 : cycles;
  if (c > kWaitCycles) c = kWaitCycles;
  k_debug_wait<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<int*>(workspace), c);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "k_debug_wait launch");
  return FLINT_OK;
}

}  // extern "C"
