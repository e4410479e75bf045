// mma_path.cuh -- the batch >= 32 layer path on the 5th-generation tensor cores.
//
// Kernels, chained with programmatic dependent launch:
//   k_router_only / k_topk  router logits, top-k and gates (layer_kernels.cuh)
//   k_mma_group     one CTA: expert histogram and token permutation -- the
//                   active experts in ascending id order (shared expert last)
//                   and, per expert, its (token, slot) pairs in token order
//   k_mma_prep      the gathered activation rows in pair order, the MMA's B
//                   operand: NVFP4 weights -> f16 rows x*sigma_t (sigma_t a
//                   power of two per token, |x*sigma_t| <= 2^15); bf16 weights
//                   -> the bf16 rows as they are
//   k_mma_ffn<GATEUP>  persistent: work item (active expert, 64 units = 128
//                   interleaved gate/up rows). Weights reach shared memory by
//                   TMA; NVFP4 codes and scales are dequantised to f16 (e2m1 *
//                   e4m3 is exact in f16) straight into tensor memory
//                   (tcgen05.st), where the MMA reads its A operand; bf16
//                   weight tiles are the A operand in shared memory (128-byte
//                   swizzled K-major layout); tcgen05.mma (kind::f16, M=128,
//                   N = the expert's tokens rounded up to 16, fp32 accumulators
//                   in tensor memory, double-buffered) and an epilogue warpgroup
//                   that applies the tensor scales, 1/sigma_t and SiLU*mul and
//                   writes h (fp32) in pair order
//   k_mma_hconv     h rows -> the down projection's B operand (f16 with a
//                   power-of-two scale per row for NVFP4 weights, bf16 else)
//   k_mma_ffn<DOWN> persistent: work item (active expert, 128 output rows),
//                   K = I; the epilogue writes y_pair = s_d * W_d h per (token,
//                   slot) in fp32
//   k_mma_combine   out_t = sum_j gate_tj y_(t,j) + y_(t,shared) (+ residual),
//                   fixed order, bf16
// Roles in the persistent kernels (16 warps): warp 0 issues the weights' TMA
// loads and warp 2 the activation rows' (two rings that run ahead of each
// other independently), warp 1 owns the tensor memory and issues the MMAs
// (one thread), warps 4-7 are the epilogue warpgroup (warp 4+i reads
// accumulator lanes 32i..32i+31), warps 8-15 dequantise. Every wait is bounded; a wait that gives up records
// FLINT_DEVCHECK_WAIT, raises a CTA-wide abort flag, and every role then drains
// what it started (copies in flight, MMAs committed) before the tensor memory
// is released.
#pragma once

#include <cuda.h>

#include "layer_kernels.cuh"

namespace flint {

constexpr int kMmaMaxTokens = 128;  // N of one MMA <= 128: an item's token tile
constexpr int kMmaGroupSmallT = 128;     // up to this many tokens one CTA groups the pairs
constexpr int kMmaMaxCallTokens = 16384; // tokens of one call on this path (prefill-size batches)
constexpr int kMmaWarps = 16;
constexpr int kMmaMaxStages = 16;   // ring depths are chosen per call, up to this
constexpr int kMmaRawBytes = 128 * 128 + 128 * 16;  // NVFP4 stage, 256 of K: codes (swizzled) + scales
// A pipeline slice is 128 of K (8 MMAs of K = 16): every slice costs the MMA
// thread a fixed ~0.25 us of waits, fence and commit besides its MMAs, so the
// wider slice halves that overhead per weight (64-wide slices measured ~0.3 us
// per slice of it)
constexpr int kMmaSliceK = 128;
constexpr int kMmaABytes = 128 * kMmaSliceK * 2;    // bf16 A stage: 128 rows x 128 of K (two 64-wide boxes)

enum MmaEpi { kEpiGateUp = 0, kEpiDown = 1 };

// Routing of the tensor-core path, in the workspace.
struct MmaRoute {
  int* n_active;  // [1]
  int* act;       // [E+S] active experts (routed ascending, then shared)
  int* off;       // [E+S+1] first pair of each active expert
  int* pair;      // [T*(k+S)] token << 8 | slot, grouped by expert, token order
  // token tiles: each active expert's pairs cut into runs of at most
  // kMmaMaxTokens (the MMA's N); a work item is (tile, row tile)
  int* n_tiles;   // [1]
  int* tile_a;    // [max tiles] active index of the tile's expert
  int* tile_off;  // [max tiles] first pair of the tile
  int* tile_n;    // [max tiles] pairs in the tile
  // large-T grouping scratch: per expert, a bit per token and the running
  // count of set bits before each 32-token word
  uint32_t* mask; // [E][T/32 rounded up]
  int* wpre;      // [E][T/32 rounded up]
  int* cnt;       // [E]
};

struct MmaParams {
  const uint16_t* x;        // [T][d] bf16
  const float* tscale;      // [E+S][3] (NVFP4) or null (bf16 weights: scale 1)
  const uint16_t* residual; // [T][d] or null
  uint16_t* out;            // [T][d]
  int* status;
  const int* ids;           // [T][k] from k_topk
  const float* gates;       // [T][k]
  int* ids_out;             // optional public copies
  float* gates_out;
  MmaRoute rt;
  uint16_t* xrows;          // [P][d] B operand of gate/up (pair order)
  float* xinv;              // [P] 1/sigma of each row (1 for bf16)
  float* h;                 // [P][I] fp32, pair order
  uint16_t* hrows;          // [P][I] B operand of down
  float* hinv;              // [P]
  float* y;                 // [T*(k+S)][d] fp32, row t*(k+S)+slot
  int T, d, I, E, k, S;
  int nvfp4;                // 1: NVFP4 weights, f16 operands; 0: bf16 weights, bf16 operands
  int n_raw, n_a, n_b;      // ring depths (raw NVFP4 stages, A stages, B stages)
  int b_bytes;              // B stage: (tokens rounded up to 64, at most 128) x 256 bytes (128 of K)
  int ksplit;               // accumulators per item (1 or 2), fed alternate K steps, summed in the epilogue
};

// ----------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst)), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16, cta_group::1.
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16, cta_group::1 (A: row i in lane
// i, two 16-bit K elements per 32-bit column).
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                           uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}
// 16 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Arrives on `bar` once every tcgen05 operation this thread issued so far is done.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}
// 16 consecutive fp32 columns of this thread's accumulator lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory operand descriptor: K-major, 128-byte swizzle, 8-row groups of
// 1024 bytes (stride dimension offset), version 1 (tcgen05).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t dsc = 0;
  dsc |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  dsc |= static_cast<uint64_t>(16 >> 4) << 16;
  dsc |= static_cast<uint64_t>(1024 >> 4) << 32;
  dsc |= static_cast<uint64_t>(1) << 46;
  dsc |= static_cast<uint64_t>(2) << 61;
  return dsc;
}
// Instruction descriptor of kind::f16: fp32 accumulate, A and B both f16 or
// both bf16, both K-major, M x N.
__host__ __device__ constexpr uint32_t mma_idesc(int M, int N, bool bf16) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Bounded wait that also gives up when another role of the CTA aborted.
__device__ __forceinline__ bool mma_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) {
      *abort_flag = 1;
      atomicOr(status, FLINT_DEVCHECK_WAIT);
      return false;
    }
  }
  return true;
}

// ----------------------------------------------------------------- router, large T
// logits [T][E] = x [T][d] . W_r^T on the register-fragment tensor cores
// (mma.sync m16n8k16, bf16 products exact, fp32 accumulation) for calls of
// many tokens, where a CUDA-core router took a third of an 8192-token call. A
// CTA computes a 64-token x 64-expert tile over K in steps of 64: both 64 x 64
// operand tiles are staged in shared memory with rows padded to 72 elements
// (the eight rows of a fragment load fall in distinct banks); warp w takes
// tokens 16*(w/2).. and experts 32*(w%2).. (four 8-expert MMA columns).
constexpr int kRtTile = 64, kRtPad = 72;

__device__ __forceinline__ void mma_bf16_m16n8k16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                  uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(256) k_router_tc(LayerParams p) {
  __shared__ __align__(16) uint16_t sx[kRtTile][kRtPad];
  __shared__ __align__(16) uint16_t sw[kRtTile][kRtPad];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = blockIdx.x * kRtTile, e0 = blockIdx.y * kRtTile, D = p.d;
  const int mt = warp >> 1, nh = warp & 1, g = lane >> 2, t4 = lane & 3;
  float acc[4][4] = {};
  auto ld32 = [](const uint16_t* q) { return *reinterpret_cast<const uint32_t*>(q); };
  for (int k0 = 0; k0 < D; k0 += kRtTile) {
    for (int c = tid; c < kRtTile * kRtTile / 8; c += blockDim.x) {  // 16-byte chunks of both tiles
      const int r = c >> 3, q = c & 7;
      uint4 vx = make_uint4(0u, 0u, 0u, 0u), vw = make_uint4(0u, 0u, 0u, 0u);
      if (t0 + r < p.T) vx = __ldg(reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(t0 + r) * D + k0) + q);
      if (e0 + r < p.E) vw = __ldg(reinterpret_cast<const uint4*>(p.wr + static_cast<size_t>(e0 + r) * D + k0) + q);
      *reinterpret_cast<uint4*>(&sx[r][8 * q]) = vx;
      *reinterpret_cast<uint4*>(&sw[r][8 * q]) = vw;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kRtTile; kk += 16) {
      const int ra = 16 * mt + g;
      const uint32_t a0 = ld32(&sx[ra][kk + 2 * t4]), a1 = ld32(&sx[ra + 8][kk + 2 * t4]);
      const uint32_t a2 = ld32(&sx[ra][kk + 8 + 2 * t4]), a3 = ld32(&sx[ra + 8][kk + 8 + 2 * t4]);
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        const int rb = 32 * nh + 8 * n + g;
        mma_bf16_m16n8k16(acc[n], a0, a1, a2, a3, ld32(&sw[rb][kk + 2 * t4]), ld32(&sw[rb][kk + 8 + 2 * t4]));
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int n = 0; n < 4; ++n) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int t = t0 + 16 * mt + g + 8 * (r >> 1), e = e0 + 32 * nh + 8 * n + 2 * t4 + (r & 1);
      if (t < p.T && e < p.E) p.logits[static_cast<size_t>(t) * p.E + e] = acc[n][r];
    }
  }
}

// ----------------------------------------------------------------- grouping
// One CTA of 512 threads (E <= 1024, T <= 128).
__global__ void __launch_bounds__(512) k_mma_group(MmaParams p) {
  __shared__ int s_ids[kMmaMaxTokens * kMaxTopK];
  __shared__ __align__(8) uint8_t s_scratch[20 * kMaxExperts];
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, TK = p.T * p.k;
  for (int i = tid; i < TK; i += blockDim.x) {
    s_ids[i] = p.ids[i];
    if (p.ids_out != nullptr) {
      p.ids_out[i] = p.ids[i];
      p.gates_out[i] = p.gates[i];
    }
  }
  __syncthreads();
  __shared__ int s_nrouted;
  cta_grouping(s_ids, p.T, p.k, p.E, p.S, p.rt.act, p.rt.off, p.rt.pair, &s_nrouted, p.rt.n_active, s_scratch,
               p.status);
  // at most kMmaGroupSmallT tokens: one token tile per active expert
  const int na = *p.rt.n_active;
  for (int a = tid; a < na; a += blockDim.x) {
    p.rt.tile_a[a] = a;
    p.rt.tile_off[a] = p.rt.off[a];
    p.rt.tile_n[a] = p.rt.off[a + 1] - p.rt.off[a];
  }
  if (tid == 0) *p.rt.n_tiles = na;
}

// ----------------------------------------------------------------- grouping, large T
// For calls of more than kMmaGroupSmallT tokens (prefill-size batches) the
// grouping is a counting sort that keeps token order, in five kernels:
//   k_grp_zero     clears the per-expert token bitmasks and counts
//   k_grp_mask     each routed (token, slot) pair sets its token's bit in its
//                  expert's mask and counts once for its expert
//   k_grp_scan     per expert (one warp): the number of set bits before each
//                  32-token word of its mask
//   k_grp_final    one CTA: active experts in ascending id (shared last), their
//                  first pair, each expert's first pair by id, and the token
//                  tiles (runs of at most kMmaMaxTokens pairs of one expert)
//   k_grp_scatter  each pair's place: its expert's first pair + the set bits of
//                  its expert's mask before its token
// A token selects an expert at most once, so its bit is its pair's rank.
__device__ __forceinline__ int grp_words(int T) { return (T + 31) >> 5; }

__global__ void __launch_bounds__(256) k_grp_zero(MmaParams p) {
  pdl_wait();  // the previous call's scatter has read the masks
  pdl_trigger();
  const int W = grp_words(p.T);
  const int n = p.E * W;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) p.rt.mask[i] = 0u;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < p.E; i += gridDim.x * blockDim.x) p.rt.cnt[i] = 0;
}

__global__ void __launch_bounds__(256) k_grp_mask(MmaParams p) {
  pdl_wait();
  pdl_trigger();
  const int W = grp_words(p.T), n = p.T * p.k;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int e = p.ids[i], t = i / p.k;
    if (p.ids_out != nullptr) {
      p.ids_out[i] = e;
      p.gates_out[i] = p.gates[i];
    }
    if (e < 0 || e >= p.E) {
      atomicOr(p.status, FLINT_DEVCHECK_EXPERT_ID);
      continue;
    }
    atomicOr(p.rt.mask + static_cast<size_t>(e) * W + (t >> 5), 1u << (t & 31));
    atomicAdd(p.rt.cnt + e, 1);
  }
}

__global__ void __launch_bounds__(256) k_grp_scan(MmaParams p) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31, e = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (e >= p.E) return;
  const int W = grp_words(p.T);
  const uint32_t* m = p.rt.mask + static_cast<size_t>(e) * W;
  int* pre = p.rt.wpre + static_cast<size_t>(e) * W;
  int run = 0;
  for (int w0 = 0; w0 < W; w0 += 32) {
    const int w = w0 + lane;
    const int c = w < W ? __popc(m[w]) : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (w < W) pre[w] = run + incl - c;
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
}

// Exclusive scan of one int per thread over a CTA of up to 1024 threads.
__device__ __forceinline__ int cta_exclusive_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? s_warp[lane] : 0;
    const int x = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += u;
    }
    if (lane < nw) s_warp[lane] = w - x;
    if (lane == 31) *total = w;
  }
  __syncthreads();
  const int r = s_warp[warp] + incl - v;
  __syncthreads();
  return r;
}

// One CTA of 1024 threads; E <= 1024.
__global__ void __launch_bounds__(1024) k_grp_final(MmaParams p) {
  __shared__ int s_warp[32];
  __shared__ int s_tot_pairs, s_tot_act, s_tot_tiles;
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, E = p.E;
  const int c = tid < E ? p.rt.cnt[tid] : 0;
  const int base = cta_exclusive_scan(c, s_warp, &s_tot_pairs);   // expert's first pair (by id)
  const int ai = cta_exclusive_scan(c > 0 ? 1 : 0, s_warp, &s_tot_act);  // active index
  const int nr = s_tot_act, routed = s_tot_pairs;
  if (tid < E) {
    p.rt.cnt[tid] = base;
    if (c > 0) {
      p.rt.act[ai] = tid;
      p.rt.off[ai] = base;
    }
  }
  if (tid < p.S) {
    p.rt.act[nr + tid] = E + tid;
    p.rt.off[nr + tid] = routed + tid * p.T;
  }
  if (tid == 0) {
    p.rt.off[nr + p.S] = routed + p.S * p.T;
    *p.rt.n_active = nr + p.S;
  }
  for (int i = tid; i < p.S * p.T; i += blockDim.x)  // the shared experts' pairs, every token
    p.rt.pair[routed + i] = ((i % p.T) << 8) | (p.k + i / p.T);
  // token tiles of each active expert (routed: thread per expert id; shared:
  // threads E.. E+S-1 stand for them)
  const bool has = (tid < E && c > 0) || (tid >= E && tid < E + p.S);
  const int a = tid < E ? ai : nr + (tid - E);
  const int npairs = tid < E ? c : p.T;
  const int ntt = has ? (npairs + kMmaMaxTokens - 1) / kMmaMaxTokens : 0;
  const int t0 = cta_exclusive_scan(ntt, s_warp, &s_tot_tiles);
  const int first = tid < E ? base : routed + (tid - E) * p.T;
  for (int j = 0; j < ntt; ++j) {
    p.rt.tile_a[t0 + j] = a;
    p.rt.tile_off[t0 + j] = first + j * kMmaMaxTokens;
    p.rt.tile_n[t0 + j] = min(kMmaMaxTokens, npairs - j * kMmaMaxTokens);
  }
  if (tid == 0) *p.rt.n_tiles = s_tot_tiles;
}

__global__ void __launch_bounds__(256) k_grp_scatter(MmaParams p) {
  pdl_wait();
  pdl_trigger();
  const int W = grp_words(p.T), n = p.T * p.k, k = p.k;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int e = p.ids[i], t = i / k;
    if (e < 0 || e >= p.E) continue;
    const size_t wi = static_cast<size_t>(e) * W + (t >> 5);
    const int pos = p.rt.cnt[e] + p.rt.wpre[wi] + __popc(p.rt.mask[wi] & ((1u << (t & 31)) - 1u));
    p.rt.pair[pos] = (t << 8) | (i - t * k);
  }
}

// ----------------------------------------------------------------- B rows of gate/up
// Warp per pair row: x[token] (bf16) -> f16 * sigma_t (NVFP4) or bf16 copy.
__global__ void __launch_bounds__(256) k_mma_prep(MmaParams p) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int P = p.T * (p.k + p.S), d = p.d;
  for (int q = blockIdx.x * 8 + (threadIdx.x >> 5); q < P; q += gridDim.x * 8) {
    const int tok = p.rt.pair[q] >> 8;
    const uint4* src = reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(tok) * d);
    uint4* dst = reinterpret_cast<uint4*>(p.xrows + static_cast<size_t>(q) * d);
    if (!p.nvfp4) {
      for (int i = lane; i < d / 8; i += 32) dst[i] = __ldg(src + i);
      if (lane == 0) p.xinv[q] = 1.f;
      continue;
    }
    float amax = 0.f;
    for (int i = lane; i < d / 8; i += 32) {
      const uint4 v = __ldg(src + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        amax = fmaxf(amax, fmaxf(fabsf(bf16_bits_to_f32(w[j] & 0xFFFFu)), fabsf(__uint_as_float(w[j] & 0xFFFF0000u))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sg = pow2_scale_for(amax);
    for (int i = lane; i < d / 8; i += 32) {
      const uint4 v = __ldg(src + i);
      uint4 o;
      o.x = bf16x2_to_f16x2_scaled(v.x, sg);
      o.y = bf16x2_to_f16x2_scaled(v.y, sg);
      o.z = bf16x2_to_f16x2_scaled(v.z, sg);
      o.w = bf16x2_to_f16x2_scaled(v.w, sg);
      dst[i] = o;
    }
    if (lane == 0) p.xinv[q] = 1.f / sg;
  }
}

// ----------------------------------------------------------------- B rows of down
// Warp per pair row: h (fp32) -> f16 * sigma_row (NVFP4) or bf16.
__global__ void __launch_bounds__(256) k_mma_hconv(MmaParams p) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int P = p.T * (p.k + p.S), I = p.I;
  for (int q = blockIdx.x * 8 + (threadIdx.x >> 5); q < P; q += gridDim.x * 8) {
    const float4* src = reinterpret_cast<const float4*>(p.h + static_cast<size_t>(q) * I);
    uint2* dst = reinterpret_cast<uint2*>(p.hrows + static_cast<size_t>(q) * I);
    float sg = 1.f;
    if (p.nvfp4) {
      float amax = 0.f;
      for (int i = lane; i < I / 4; i += 32) {
        const float4 v = __ldcg(src + i);
        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      sg = pow2_scale_for(amax);
    }
    for (int i = lane; i < I / 4; i += 32) {
      const float4 v = __ldcg(src + i);
      uint2 o;
      if (p.nvfp4) {
        o.x = pack_f16x2(v.x * sg, v.y * sg);
        o.y = pack_f16x2(v.z * sg, v.w * sg);
      } else {
        const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
        o.x = *reinterpret_cast<const uint32_t*>(&a);
        o.y = *reinterpret_cast<const uint32_t*>(&b);
      }
      dst[i] = o;
    }
    if (lane == 0) p.hinv[q] = 1.f / sg;
  }
}

// ----------------------------------------------------------------- combine
// Thread per 8 outputs: fixed slot order 0..k-1, then the shared expert.
__global__ void __launch_bounds__(256) k_mma_combine(MmaParams p) {
  pdl_wait();
  pdl_trigger();
  const int KS = p.k + p.S, d8 = p.d / 8;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= p.T * d8) return;
  const int t = idx / d8, c = idx % d8;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  for (int j = 0; j < KS; ++j) {
    const float g = (j < p.k) ? p.gates[t * p.k + j] : 1.f;
    const float4* yr = reinterpret_cast<const float4*>(p.y + static_cast<size_t>(t * KS + j) * p.d + 8 * c);
    const float4 a = __ldcg(yr), b = __ldcg(yr + 1);
    acc[0] = fmaf(g, a.x, acc[0]);
    acc[1] = fmaf(g, a.y, acc[1]);
    acc[2] = fmaf(g, a.z, acc[2]);
    acc[3] = fmaf(g, a.w, acc[3]);
    acc[4] = fmaf(g, b.x, acc[4]);
    acc[5] = fmaf(g, b.y, acc[5]);
    acc[6] = fmaf(g, b.z, acc[6]);
    acc[7] = fmaf(g, b.w, acc[7]);
  }
  const size_t o = static_cast<size_t>(t) * p.d + 8 * c;
  if (p.residual != nullptr) {
    const uint4 r = __ldg(reinterpret_cast<const uint4*>(p.residual + o));
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      acc[2 * j] += bf16_bits_to_f32(w[j] & 0xFFFFu);
      acc[2 * j + 1] += __uint_as_float(w[j] & 0xFFFF0000u);
    }
  }
  uint4 ov;
  uint32_t* ow = reinterpret_cast<uint32_t*>(&ov);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * j], acc[2 * j + 1]);
    ow[j] = *reinterpret_cast<const uint32_t*>(&b);
  }
  *reinterpret_cast<uint4*>(p.out + o) = ov;
}

// ----------------------------------------------------------------- the tensor-core FFN kernel
// Tensor maps of one call. Raw NVFP4: codes [experts][rows][K/2] bytes, box
// (128 B, 128 rows, 1), 128-byte swizzle; scales [experts][rows][K/16], box
// (16 B, 128, 1). bf16 weights: [experts][rows][K] bf16, box (64, 128, 1),
// 128-byte swizzle. B rows: [P][K] 16-bit, box (64, 64), 128-byte swizzle.
struct MmaMaps {
  CUtensorMap codes;
  CUtensorMap scales;
  CUtensorMap brows;
};

// Dequantise one half (32 elements) of a 64-element slice of K of the 128-row
// A tile straight into tensor memory (NVFP4 weights): the warp owns the lanes
// of its quarter (rows 32*qtr..+31, qtr = warp % 4): 32 codes and their 2
// scales of its row -> 16 columns of two f16 values each. The operand never
// passes through shared memory.
__device__ __forceinline__ void dequant_slice_tmem(const uint8_t* raw, int sub, uint32_t a_tmem, int qtr, int half,
                                                   int lane) {
  const int r = 32 * qtr + lane;
  const int chunk = 2 * sub + half;  // 16-byte code chunk of the 128-byte raw row
  const uint4 cv = lds128(raw + r * 128 + ((chunk ^ (r & 7)) << 4));
  const uint32_t s2 = *reinterpret_cast<const uint16_t*>(raw + 128 * 128 + r * 16 + 4 * sub + 2 * half);
  uint32_t sh;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(sh) : "h"(static_cast<uint16_t>(s2)));
  const __half2 hs = *reinterpret_cast<const __half2*>(&sh);
  const __half2 sc[2] = {__low2half2(hs), __high2half2(hs)};
  const uint32_t cw[4] = {cv.x, cv.y, cv.z, cv.w};
  uint32_t out[16];
#pragma unroll
  for (int q = 0; q < 4; ++q) {  // 8 elements per q; words 0,1 -> block 0, words 2,3 -> block 1
    uint32_t f[4];
    e2m1x8_to_f16x2(cw[q], *reinterpret_cast<uint32_t(*)[4]>(&f[0]));
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __half2 v = __hmul2(*reinterpret_cast<const __half2*>(&f[j]), sc[q >> 1]);
      out[4 * q + j] = *reinterpret_cast<const uint32_t*>(&v);
    }
  }
  tmem_st16(a_tmem + (static_cast<uint32_t>(32 * qtr) << 16) + static_cast<uint32_t>(16 * half), out);
}

template <int EPI>
__global__ void __launch_bounds__(kMmaWarps * 32, 1)
    k_mma_ffn(MmaParams p, const __grid_constant__ MmaMaps maps, int ncols) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t raw_full[kMmaMaxStages], raw_empty[kMmaMaxStages];
  // A and B stages advance together (one of each per 64-wide K slice, rings
  // of the same depth), so one barrier says both of a slot are free
  __shared__ __align__(8) uint64_t a_full[kMmaMaxStages], b_full[kMmaMaxStages], ab_empty[kMmaMaxStages];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], mma_done;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_nact;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool fp4 = p.nvfp4 != 0;
  const int NR = p.n_raw, NA = p.n_a, BB = p.b_bytes;  // p.n_b == p.n_a
  // MMA issuers: with two accumulators per item, each has its own thread
  // (warps 1 and 3), issuing the K steps of its accumulator (a thread takes
  // ~60 ns per tcgen05.mma, more than the MMA itself at these N)
  const int NI = p.ksplit;
  // 1024-aligned carve-up: [raw stages (NVFP4 only)][A stages][B stages]
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* raw = base;
  uint8_t* abuf = raw + (fp4 ? NR * kMmaRawBytes : 0);  // bf16 weights: A stages in shared memory
  uint8_t* bbuf = abuf + (fp4 ? 0 : NA * kMmaABytes);
  // tensor memory: two accumulators (columns 0..255), then the NVFP4 A stages
  // (32 columns each: 128 rows x 64 of K in f16)
  constexpr uint32_t kAccCols = 2 * kMmaMaxTokens;
  const int K = EPI == kEpiGateUp ? p.d : p.I;
  const int tiles = EPI == kEpiGateUp ? p.I / 64 : p.d / 128;
  const int n_sub = K / kMmaSliceK;
  const int KS = p.k + p.S;
  // With two accumulators, issuer i takes the slices s = i (mod 2), all eight
  // K steps of each: one commit per slice (a commit costs the issuing thread
  // about as much as four MMAs). With a single slice both take alternate K
  // steps of it.
  const bool SLICE_SPLIT = NI == 2 && n_sub >= 2;

  if (tid == 0) {
    for (int i = 0; i < kMmaMaxStages; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_empty[i], 8);
      mbar_init(&a_full[i], fp4 ? 4 : 1);
      mbar_init(&b_full[i], 1);
      mbar_init(&ab_empty[i], SLICE_SPLIT ? 1 : NI);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], NI);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(&mma_done, NI);
    fence_barrier_init();
    s_abort = 0;
  }
  if (warp == 1) tmem_alloc(&s_tmem, static_cast<uint32_t>(ncols));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  if (tid == 0) s_nact = p.rt.n_tiles[0];
  __syncthreads();
  pdl_trigger();
  const uint32_t tmem = s_tmem;
  const int n_items = s_nact * tiles;  // (token tile, row tile)
  volatile int* abort_flag = &s_abort;
  // on abort: wait (bounded) for every copy a producer started; stages older
  // than the ring depth were consumed, so they have landed
  auto drain = [&](uint64_t* full, int ns, int n) {
    for (int i = max(0, n - ns); i < n; ++i) mbar_wait(&full[i % ns], (i / ns) & 1, p.status);
  };

  // The producers issue a stage's operations from several lanes at once (the
  // barrier's byte count from lane 0, each copy from a lane of its own): one
  // thread takes ~0.25 us per operation. Every lane waits for the slot; the
  // warp goes on only if all lanes saw it free.
  if (warp == 0) {
    // ------------------------------------------------ A producer: weights
    int rc = 0, ac = 0;  // stages issued: raw NVFP4, A (bf16 weights)
    bool ok = true;
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
      const int tt = it / tiles, t = it % tiles;  // token tile, row tile
      const int e = p.rt.act[p.rt.tile_a[tt]];
      for (int s = 0; s < n_sub && ok; ++s) {
        if (fp4) {
          if ((s & 1) != 0) continue;
          const int slot = rc % NR;
          if (!(ok = __all_sync(0xffffffffu, mma_wait(&raw_empty[slot], ((rc / NR) & 1) ^ 1, abort_flag, p.status))))
            break;
          uint8_t* st = raw + slot * kMmaRawBytes;
          if (lane == 0) mbar_arrive_expect_tx(&raw_full[slot], kMmaRawBytes);
          else if (lane == 1) tma_load_3d(st, &maps.codes, (s / 2) * 128, t * 128, e, &raw_full[slot]);
          else if (lane == 2) tma_load_3d(st + 128 * 128, &maps.scales, (s / 2) * 16, t * 128, e, &raw_full[slot]);
          ++rc;
        } else {
          const int slot = ac % NA;
          if (!(ok = __all_sync(0xffffffffu, mma_wait(&ab_empty[slot], ((ac / NA) & 1) ^ 1, abort_flag, p.status))))
            break;
          if (lane == 0) mbar_arrive_expect_tx(&a_full[slot], kMmaABytes);
          else if (lane <= 2)  // the slice's two 64-wide K boxes
            tma_load_3d(abuf + slot * kMmaABytes + (lane - 1) * (kMmaABytes / 2), &maps.codes,
                        s * kMmaSliceK + (lane - 1) * 64, t * 128, e, &a_full[slot]);
          ++ac;
        }
      }
    }
    if (!ok && lane == 0) {
      drain(raw_full, NR, rc);
      drain(a_full, NA, ac);
    }
  } else if (warp == 2) {
    // ------------------------------------------------ B producer: activation rows
    int bc = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
      const int tt = it / tiles;
      const int off = p.rt.tile_off[tt], nt = p.rt.tile_n[tt];
      const int npad = (nt + 15) & ~15;
      for (int s = 0; s < n_sub && ok; ++s) {
        const int slot = bc % NA;
        if (!(ok = __all_sync(0xffffffffu, mma_wait(&ab_empty[slot], ((bc / NA) & 1) ^ 1, abort_flag, p.status))))
          break;
        // 64-row boxes (rows past the expert's tokens are loaded but not
        // multiplied; rows past the last pair are zero-filled)
        const int nbox = (npad + 63) / 64;
        // two 64-wide K halves of the slice, each [rows][128 B] (half h at BB / 2 * h)
        if (lane == 0) mbar_arrive_expect_tx(&b_full[slot], 2 * nbox * 8192);
        else if (lane <= 2 * nbox) {
          const int h = (lane - 1) / nbox, j = (lane - 1) % nbox;
          tma_load_2d(bbuf + slot * BB + h * (BB / 2) + j * 8192, &maps.brows, s * kMmaSliceK + 64 * h, off + 64 * j,
                      &b_full[slot]);
        }
        ++bc;
      }
    }
    if (!ok && lane == 0) drain(b_full, NA, bc);
  } else if (warp == 1 || (warp == 3 && NI == 2)) {
    // ------------------------------------------------ MMA issuers
    if (lane == 0) {
      const int iss = warp == 1 ? 0 : 1;  // accumulator (its slices, or alternate K steps of one)
      int sc = 0, icount = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++icount) {
        const int nt = p.rt.tile_n[it / tiles];
        const int npad = (nt + 15) & ~15;
        const uint32_t idesc = mma_idesc(128, npad, !fp4);
        const int ab = icount & 1;
        if (!(ok = mma_wait(&acc_empty[ab], ((icount >> 1) & 1) ^ 1, abort_flag, p.status))) break;
        tc_fence_after();
        // the NI accumulators of an item are kMmaMaxTokens / NI columns apart;
        // independent accumulation chains, summed in the epilogue
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(ab * kMmaMaxTokens + iss * (kMmaMaxTokens / NI));
        const int k0 = SLICE_SPLIT ? 0 : iss, kstep = SLICE_SPLIT ? 1 : NI;
        bool first = true;  // the accumulator's first MMA of the item overwrites it
        for (int s = 0; s < n_sub; ++s) {
          const int as = sc % NA;
          if (SLICE_SPLIT && (s & 1) != iss) {  // the other issuer's slice
            ++sc;
            continue;
          }
          if (!(ok = mma_wait(&a_full[as], (sc / NA) & 1, abort_flag, p.status))) break;
          if (!(ok = mma_wait(&b_full[as], (sc / NA) & 1, abort_flag, p.status))) break;
          tc_fence_after();
          const uint32_t baddr = smem_addr(bbuf + as * BB);
          if (fp4) {
            const uint32_t a_tmem = tmem + kAccCols + static_cast<uint32_t>(64 * as);
            for (int kk = k0; kk < 8; kk += kstep) {
              mma_f16_ts(d_tmem, a_tmem + 8 * kk, sw128_desc(baddr + (kk >> 2) * (BB / 2) + 32 * (kk & 3)), idesc,
                         first ? 0u : 1u);
              first = false;
            }
          } else {
            const uint32_t aaddr = smem_addr(abuf + as * kMmaABytes);
            for (int kk = k0; kk < 8; kk += kstep) {
              mma_f16(d_tmem, sw128_desc(aaddr + (kk >> 2) * (kMmaABytes / 2) + 32 * (kk & 3)),
                      sw128_desc(baddr + (kk >> 2) * (BB / 2) + 32 * (kk & 3)), idesc, first ? 0u : 1u);
              first = false;
            }
          }
          mma_commit(&ab_empty[as]);
          ++sc;
        }
        if (ok) mma_commit(&acc_full[ab]);
      }
      // every MMA of both issuers completes before tensor memory is freed
      mma_commit(&mma_done);
      mbar_wait(&mma_done, 0, p.status);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------ epilogue warpgroup
    const int ew = warp - 4, m = 32 * ew + lane;  // accumulator lane = A tile row
    int icount = 0;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x, ++icount) {
      const int tt = it / tiles, t = it % tiles;
      const int e = p.rt.act[p.rt.tile_a[tt]];
      const int off = p.rt.tile_off[tt], nt = p.rt.tile_n[tt];
      const int ab = icount & 1;
      if (!mma_wait(&acc_full[ab], (icount >> 1) & 1, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * ew) << 16) + static_cast<uint32_t>(ab * kMmaMaxTokens);
      if (EPI == kEpiGateUp) {
        const float sgt = fp4 ? __ldg(p.tscale + 3 * e + 0) : 1.f, sut = fp4 ? __ldg(p.tscale + 3 * e + 1) : 1.f;
        const int unit = t * 64 + (m >> 1);
        for (int c0 = 0; c0 < nt; c0 += 16) {
          // column scales: lane j (mod 16) loads column c0 + j, then broadcasts
          const float xin = (c0 + (lane & 15) < nt) ? p.xinv[off + c0 + (lane & 15)] : 0.f;
          float v[16];
          tmem_ld16(taddr + c0, v);
          if (p.ksplit > 1) {
            float v2[16];
            tmem_ld16(taddr + kMmaMaxTokens / 2 + c0, v2);
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] += v2[j];
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float other = __shfl_xor_sync(0xffffffffu, v[j], 1);
            const float xi = __shfl_sync(0xffffffffu, xin, j);
            const int n = c0 + j;
            if ((m & 1) == 0 && n < nt)
              p.h[static_cast<size_t>(off + n) * p.I + unit] = swiglu(v[j] * sgt * xi, other * sut * xi);
          }
        }
      } else {
        const float sdt = fp4 ? __ldg(p.tscale + 3 * e + 2) : 1.f;
        const int row = t * 128 + m;
        for (int c0 = 0; c0 < nt; c0 += 16) {
          const bool in = c0 + (lane & 15) < nt;
          const float hin = in ? p.hinv[off + c0 + (lane & 15)] : 0.f;
          const int prn = in ? p.rt.pair[off + c0 + (lane & 15)] : 0;
          float v[16];
          tmem_ld16(taddr + c0, v);
          if (p.ksplit > 1) {
            float v2[16];
            tmem_ld16(taddr + kMmaMaxTokens / 2 + c0, v2);
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] += v2[j];
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = c0 + j;
            const float hi = __shfl_sync(0xffffffffu, hin, j);
            const int pr = __shfl_sync(0xffffffffu, prn, j);
            if (n < nt) {
              const int yrow = (pr >> 8) * KS + (pr & 0xFF);
              p.y[static_cast<size_t>(yrow) * p.d + row] = v[j] * sdt * hi;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
    }
  } else if (warp >= 8 && fp4) {
    // ------------------------------------------------ dequantisers (NVFP4)
    // two groups of four warps (one per tensor-memory lane quarter) take the
    // even and the odd slices, so that two slices are converted at once; a
    // warp converts both halves of its slices' K for its quarter
    const int grp = (warp - 8) >> 2, qtr = warp & 3;
    int rc = 0, sc = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
      for (int s = 0; s < n_sub; ++s) {
        const int rs = rc % NR, as = sc % NA;
        if ((s & 1) == grp) {
          if (!(ok = mma_wait(&raw_full[rs], (rc / NR) & 1, abort_flag, p.status))) break;
          if (!(ok = mma_wait(&ab_empty[as], ((sc / NA) & 1) ^ 1, abort_flag, p.status))) break;
          tc_fence_after();  // the stage's previous MMAs are done before it is rewritten
          const uint32_t a_tmem = tmem + kAccCols + static_cast<uint32_t>(64 * as);
#pragma unroll
          for (int sub2 = 0; sub2 < 2; ++sub2) {  // the slice's two 64-wide sub-slices of the raw stage
            dequant_slice_tmem(raw + rs * kMmaRawBytes, 2 * (s & 1) + sub2, a_tmem + 32 * sub2, qtr, 0, lane);
            dequant_slice_tmem(raw + rs * kMmaRawBytes, 2 * (s & 1) + sub2, a_tmem + 32 * sub2, qtr, 1, lane);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&a_full[as]);
        }
        ++sc;
        if ((s & 1) == 1) {  // both groups are done with this raw stage (two slices)
          if (lane == 0) mbar_arrive(&raw_empty[rs]);
          ++rc;
        }
      }
    }
  }
  // ------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(ncols));
  }
}

}  // namespace flint
