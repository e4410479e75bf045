// fused_layer.cuh -- the whole layer in one persistent kernel (batch <= 8).
//
// One CTA per SM (16 warps), every SM busy in every phase:
//   P0  bulk copies of this CTA's router rows and of each warp's slice of
//       the shared expert's gate/up units; L2 prefetch of this CTA's block of
//       the shared expert's down rows
//   P1  per-token scales, x converted once to f16 (lane-interleaved), router
//       logits ((row, token) tasks over the warps), stored as tagged 64-bit
//       words (launch tag | logit) in 8 replicas
//   P2  every CTA: top-k of every token (a warp per token waits until all E
//       logits carry this launch's tag, then selects) and the token grouping,
//       kept in shared memory
//   P3  gate/up through per-warp bulk-copy rings: first the warp's shared-
//       expert units, then its range of the routed experts' units (split by
//       compute cost); h written as tagged 64-bit words; L2 prefetch of this
//       CTA's block of down rows of every routed expert
//   P4  every h row polled until all its values carry this launch's tag, then
//       converted once per CTA to f16 (power-of-two scale per row) in shared
//       memory; down rows of this CTA's block streamed through per-warp rings,
//       fixed-order gated combine (+ residual)
// The launch tag comes from a generation word in the workspace control block
// that CTA 0 advances once it has seen every h row (by then every CTA has read
// the generation). There is no grid barrier: the two cross-CTA dependencies
// (all logits before top-k, all h before the down phase) are the tagged
// words themselves. Every wait is bounded (FLINT_DEVCHECK_WAIT). The launch is
// cooperative, so every CTA is resident.
//
// The tensor-core variant (TC = true, used at 2..8 tokens) keeps P0-P2 and the
// h exchange and replaces the CUDA-core inner loops of P3 and P4 with
// register-fragment mma.sync (fused_tc.cuh): gate/up work is split into tiles
// of 8 units (16 rows) of one expert, each tile's K range into two halves
// ("items", d >= 1024) taken by adjacent warps of the same CTA and summed in
// shared memory (two partial sums, so the float sum does not depend on their
// order); each item streams 512-column stages of its 16 rows through the
// warp's ring as 2-D TMA boxes (128-byte swizzle). The down phase computes 16
// rows of the CTA's block per active expert with the same fragments.
#pragma once

#include <cuda.h>

#include "layer_kernels.cuh"
#include "fused_tc.cuh"

namespace flint {

constexpr int kFusedMaxTokens = 8;
constexpr int kTcMinTokens = 2;      // the tensor-core variant is the default from this batch
constexpr int kFusedWarps = 16;
constexpr int kFusedDownTokens = 4;   // tokens per pass in the down phase
// Tagged logits are written to this many replicas; CTA c reads replica c % R,
// so each line is polled by G/R CTAs instead of all of them.
constexpr int kLogitReplicas = 8;

// Tensor maps of the tensor-core variant over the gate/up rows of all experts:
// codes [E+S][2*inter][d/2] bytes, box 128 x 16 (128-byte swizzle); block
// scales [E+S][2*inter][d/16] bytes, box 32 x 16.
struct FusedMaps {
  CUtensorMap codes;
  CUtensorMap scales;
};

__device__ __forceinline__ unsigned ld_relaxed_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Exclusive prefix over the active experts of the gate/up cost of expert a,
// I units x ceil(tokens / tg) passes, computed by one warp into cost[0..n].
__device__ __forceinline__ void cost_prefix(const RouteDesc* dsc, int n_active, int I, int tg, int* cost, int lane) {
  const int per = (n_active + 31) / 32;
  int cnt = 0;
  for (int i = 0; i < per; ++i) {
    const int a = lane * per + i;
    if (a < n_active) cnt += I * ((dsc->off[a + 1] - dsc->off[a] + tg - 1) / tg);
  }
  int ex = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, ex, o);
    if (lane >= o) ex += v;
  }
  ex -= cnt;
  for (int i = 0; i < per; ++i) {
    const int a = lane * per + i;
    if (a < n_active) {
      cost[a] = ex;
      ex += I * ((dsc->off[a + 1] - dsc->off[a] + tg - 1) / tg);
    }
  }
  if (lane == 31) cost[n_active] = ex;
}

// Down rows of one staged block (up to 4*RPS rows, RPS = rows per warp step)
// against TG tokens' h (16 f16x2 registers each): each lane accumulates its
// 32-column slice for all 4 steps x TG tokens, then one transposed butterfly
// per row group (VRD lanes) reduces them. out[g] is the total of value index
// g*VRD + (lane % VRD) (value index = step*TG + token) when 4*TG > VRD, else
// out[0] is the total of index (lane % VRD) >> log2(VRD / (4*TG)).
template <int I, int TG>
__device__ __forceinline__ void down_block(const uint8_t* st, int roff, int rows, const uint32_t* hh, int lane,
                                           float* out) {
  constexpr int VRD = I / 32, RPS = 32 / VRD, ROWC = I / 2, ROWS = I / 16, V = 4 * TG;
  const int rs = lane / VRD, cbk = lane % VRD;
  float v[V];
#pragma unroll
  for (int step = 0; step < 4; ++step) {
    const int row = step * RPS + rs;
    float acc[TG];
#pragma unroll
    for (int t = 0; t < TG; ++t) acc[t] = 0.f;
    if (row < rows) {
      const uint4 cv = lds128(st + row * ROWC + cbk * 16);
      const uint32_t s2 = *reinterpret_cast<const uint16_t*>(st + roff + row * ROWS + cbk * 2);
      dot32_strided<TG, 16>(cv, s2, hh, acc);
    }
#pragma unroll
    for (int t = 0; t < TG; ++t) v[step * TG + t] = acc[t];
  }
  if constexpr (V <= VRD) {
    out[0] = xreduce<VRD, V>(v, lane);
  } else {
#pragma unroll
    for (int g = 0; g < V / VRD; ++g) out[g] = xreduce<VRD, VRD>(v + g * VRD, lane);
  }
}

// Shared-memory bytes of the router-rows region, which later serves as the
// grouping's scratch (20 bytes per expert).
__host__ __device__ constexpr size_t fused_rows_bytes(int row_bytes, int E) {
  return ((static_cast<size_t>(row_bytes > 20 * E ? row_bytes : 20 * E)) + 127) & ~static_cast<size_t>(127);
}

// Shared-memory bytes of the down phase's h copy: R rows of I f16.
__host__ __device__ constexpr size_t fused_h16_bytes(int R, int I) {
  return ((static_cast<size_t>(R) * I * 2) + 127) & ~static_cast<size_t>(127);
}

template <int D, int I, bool TC>
__global__ void __launch_bounds__(kFusedWarps * 32, 1) k_layer(LayerParams p, const __grid_constant__ FusedMaps maps) {
  using M = GateUpMap<D>;
  constexpr int NVR = D / 256;   // router: 8-element bf16 vectors per lane
  constexpr int VRD = I / 32;    // down: 16-byte vectors per row (lanes per row)
  constexpr int RPS = 32 / VRD;  // down: rows per warp step
  constexpr int TGD = kFusedDownTokens;
  constexpr int ROWC = I / 2, ROWS = I / 16;
  constexpr int MAXR = kFusedMaxTokens * (kMaxTopK + 1);
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_ids[kFusedMaxTokens * kMaxTopK];
  __shared__ float s_gates[kFusedMaxTokens * kMaxTopK];
  __shared__ float s_sigma[kFusedMaxTokens], s_f[kFusedMaxTokens];
  __shared__ int s_cost[kFusedWarps][kFusedMaxTokens * kMaxTopK + 2];  // per-warp cost prefix over <= T*k+1 experts
  __shared__ float s_hinv[MAXR];
  __shared__ unsigned s_gen;
  __shared__ int s_fail;
  __shared__ __align__(8) uint64_t s_bar[kFusedWarps * kMaxStages + 2];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = p.T, E = p.E, k = p.k, S = p.S, KS = k + S, G = gridDim.x, c = blockIdx.x;
  const int R = T * KS;

  // ---- shared-memory carve-up: [desc][x][router rows][work]
  RouteDesc* dsc = reinterpret_cast<RouteDesc*>(smem);
  constexpr int XSTR = TC ? tc_b_stride(D) : 2 * D;  // bytes per token row of x16
  constexpr int HSTR = TC ? tc_b_stride(I) : 2 * I;  // bytes per row of h16 (down phase)
  const size_t xbytes = static_cast<size_t>(T) * XSTR;
  const size_t xpad = (xbytes + 127) & ~static_cast<size_t>(127);
  // x * sigma_t as f16, lane-interleaved: element i of token t at
  // t*D + (((i % 32) / 8) * (D / 32) + i / 32) * 8 + i % 8, so the 16-byte
  // chunks the lanes of a gate/up step read are contiguous (tensor-core
  // variant: the B-fragment order of tc_b_offset, rows XSTR bytes apart)
  uint16_t* x16 = reinterpret_cast<uint16_t*>(smem + sizeof(RouteDesc));
  uint8_t* rsm = smem + sizeof(RouteDesc) + xpad;
  const int rpc = (E + G - 1) / G;  // router rows per CTA
  uint8_t* work = rsm + fused_rows_bytes(rpc * D * 2, E);
  if constexpr (TC) work += (1024u - (smem_addr(work) & 1023u)) & 1023u;  // swizzled TMA boxes
  uint64_t* ring_bars = s_bar;                        // [warp][kMaxStages]
  uint64_t* rbar = s_bar + kFusedWarps * kMaxStages;  // router rows
  const int ns_g = p.ns_gateup, ns_d = p.ns_down;
  const int nb = p.down_nb, n0 = c * nb, nrows = max(0, min(nb, p.d - n0));
  const int r_begin = min(E, c * rpc), r_end = min(E, (c + 1) * rpc);

  // ---- P0: start the copies before anything else
  if (tid == 0) {
    for (int i = 0; i < kFusedWarps * kMaxStages + 2; ++i) mbar_init(&s_bar[i], 1);
    fence_barrier_init();
    const uint32_t rbytes = static_cast<uint32_t>(r_end - r_begin) * D * 2;
    mbar_arrive_expect_tx(rbar, rbytes);
    if (rbytes) bulk_g2s(rsm, p.wr + static_cast<size_t>(r_begin) * D, rbytes, rbar);
    s_gen = ld_relaxed_u32(p.counter + 1);
    s_fail = 0;
  } else if (tid == 32 && S > 0) {
    const long long e = E;
    if (nrows > 0) {
      prefetch_l2(p.codes + e * p.cpe + static_cast<long long>(I) * p.d + static_cast<long long>(n0) * ROWC, nrows * ROWC);
      prefetch_l2(p.scales + e * p.spe + static_cast<long long>(I) * p.d / 8 + static_cast<long long>(n0) * ROWS,
                  nrows * ROWS);
    }
  }
  __syncthreads();
  const unsigned gen = s_gen, tag = gen + 1u;

  // ---- the warp's bulk-copy ring: first the shared expert's units (they do
  // not depend on the routing, so they are fetched now), then a range of the
  // routed experts' units (after the routing step)
  uint8_t* ring = work + static_cast<size_t>(warp) * ns_g * p.stage_gateup;
  uint64_t* bars = ring_bars + warp * kMaxStages;
  int issued = 0, consumed = 0;
  auto issue_units = [&](int e, int uu, int cu, int slot) {
    uint8_t* st = ring + slot * p.stage_gateup;
    mbar_arrive_expect_tx(&bars[slot], cu * M::UNIT_BYTES);
    bulk_g2s(st, p.codes + e * p.cpe + static_cast<long long>(uu) * D, cu * M::UNIT_CODE, &bars[slot]);
    bulk_g2s(st + M::CU * M::UNIT_CODE, p.scales + e * p.spe + static_cast<long long>(uu) * (D / 8),
             cu * M::UNIT_SCALE, &bars[slot]);
  };
  const int NW = G * kFusedWarps, gw = c * kFusedWarps + warp;  // grid <= 240 CTAs (host check)
  const int sh_begin = (S > 0 && !TC) ? gw * I / NW : 0;
  const int sh_end = (S > 0 && !TC) ? (gw + 1) * I / NW : 0;
  int sh_issue = sh_begin;
  while (issued < ns_g && sh_issue < sh_end) {
    const int cu = min(M::CU, sh_end - sh_issue);
    if (lane == 0) issue_units(E, sh_issue, cu, issued % ns_g);
    sh_issue += cu;
    ++issued;
  }
  // tensor-core variant: the warp's stream of stages (16 tile rows x 512
  // columns). This CTA's local tiles are its shared-expert tiles, then its
  // range of routed tiles; item li = (local tile li / KP, K part li % KP)
  // belongs to warp li % kFusedWarps, and SPI stages make an item.
  constexpr int NTE = I / kTcUnits;        // tiles per expert
  constexpr int KP = (D >= 1024) ? 2 : 1;  // K parts (items) per tile
  constexpr int SPI = D / kTcStageK / KP;  // stages per item
  const int n_sh = S * NTE;                // shared-expert tiles (<= 128, below the grid size)
  const int shb0 = c * n_sh / G, nsh_c = (c + 1) * n_sh / G - shb0;
  int rt0 = 0;  // first routed tile of this CTA, once the routing is known
  uint8_t* tc_codes = work + static_cast<size_t>(warp) * ns_g * kTcStageCodes;
  uint8_t* tc_scales = work + static_cast<size_t>(kFusedWarps) * ns_g * kTcStageCodes +
                       static_cast<size_t>(warp) * ns_g * kTcStageScales;
  float* tc_acc = reinterpret_cast<float*>(work + static_cast<size_t>(kFusedWarps) * ns_g * (kTcStageCodes + kTcStageScales));
  int* tc_cnt = reinterpret_cast<int*>(tc_acc + static_cast<size_t>(p.tc_lt) * 128);
  auto tc_tile = [&](int lt, int& e, int& ti, int& a) {  // local tile -> expert, tile index, active slot
    if (lt < nsh_c) {
      e = E;
      ti = shb0 + lt;
      a = -1;
    } else {
      const int gt = rt0 + lt - nsh_c;
      a = gt / NTE;
      ti = gt - a * NTE;
      e = dsc->act[a];
    }
  };
  auto tc_issue = [&](int q) {  // one lane: stage q of the stream into slot q % ns_g
    const int m = q / SPI, s = q - m * SPI, li = warp + kFusedWarps * m, lt = li / KP, part = li - lt * KP;
    int e, ti, a;
    tc_tile(lt, e, ti, a);
    const int k0 = (part * SPI + s) * kTcStageK, slot = q % ns_g;
    uint8_t* cs = tc_codes + slot * kTcStageCodes;
    mbar_arrive_expect_tx(&bars[slot], kTcStageCodes + kTcStageScales);
    tma_load_3d(cs, &maps.codes, k0 / 2, 16 * ti, e, &bars[slot]);
    tma_load_3d(cs + 2048, &maps.codes, k0 / 2 + 128, 16 * ti, e, &bars[slot]);
    tma_load_3d(tc_scales + slot * kTcStageScales, &maps.scales, k0 / 16, 16 * ti, e, &bars[slot]);
  };
  if constexpr (TC) {  // the shared tiles' stages do not depend on the routing
    const int sh_items = nsh_c * KP;
    const int my_sh = warp < sh_items ? ((sh_items - 1 - warp) / kFusedWarps + 1) * SPI : 0;
    while (issued < ns_g && issued < my_sh) {
      if (lane == 0) tc_issue(issued);
      ++issued;
    }
  }

  // ---- P1: router logits first (the top-k waits for them), then token
  // statistics and the f16 copy of x the gate/up phase reads after the routing
  bool ok = true;
  // x (bf16, read-only for the whole launch) is read through the L1 cache
  const uint4* xg = reinterpret_cast<const uint4*>(p.x);
  const int n_tasks = (r_end - r_begin) * T;
  if (warp < n_tasks && ok) ok = mbar_wait(rbar, 0, p.status);
  for (int task = warp; task < n_tasks && ok; task += kFusedWarps) {
    const int r = task / T, t = task % T;
    const uint16_t* wrow = reinterpret_cast<const uint16_t*>(rsm) + static_cast<size_t>(r) * D;
    // the token's sum of squares in the same order as the statistics below,
    // so the input-norm factor is the same value
    float sum = 0.f, ss = 0.f;
#pragma unroll
    for (int i = 0; i < NVR; ++i) {
      const uint4 wv = lds128(wrow + 8 * (lane + 32 * i));
      const uint4 xv = __ldg(xg + (static_cast<size_t>(t) * D + 8 * (lane + 32 * i)) / 8);
      const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
      const uint32_t xx[4] = {xv.x, xv.y, xv.z, xv.w};
      float a = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float xa = bf16_bits_to_f32(xx[q] & 0xFFFFu), xb = __uint_as_float(xx[q] & 0xFFFF0000u);
        a = fmaf(bf16_bits_to_f32(ww[q] & 0xFFFFu), xa, a);
        a = fmaf(__uint_as_float(ww[q] & 0xFFFF0000u), xb, a);
        ss = fmaf(xa, xa, ss);
        ss = fmaf(xb, xb, ss);
      }
      sum += a;
    }
    sum = warp_sum(sum);
    ss = warp_sum(ss);
    const float irms = p.input_norm ? 1.f / sqrtf(ss / static_cast<float>(D) + kRmsEps) : 1.f;
    if (lane < kLogitReplicas)
      st_tagged(p.tlogits + (static_cast<size_t>(t) * kLogitReplicas + lane) * E + r_begin + r, tag, sum * irms);
  }
  // statistics of token t on warp kFusedWarps-1-t (idle during the router at
  // one token)
  if (kFusedWarps - 1 - warp < T && ok) {
    const int t = kFusedWarps - 1 - warp;
    float amax = 0.f, ss = 0.f;
#pragma unroll
    for (int i = 0; i < NVR; ++i) {
      const uint4 v = __ldg(xg + (static_cast<size_t>(t) * D + 8 * (lane + 32 * i)) / 8);
      const uint32_t ww[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float a = bf16_bits_to_f32(ww[q] & 0xFFFFu), b = __uint_as_float(ww[q] & 0xFFFF0000u);
        amax = fmaxf(amax, fmaxf(fabsf(a), fabsf(b)));
        ss = fmaf(a, a, ss);
        ss = fmaf(b, b, ss);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    ss = warp_sum(ss);
    const float irms = p.input_norm ? 1.f / sqrtf(ss / static_cast<float>(D) + kRmsEps) : 1.f;
    const float sg = pow2_scale_for(amax);
    if (lane == 0) {
      s_sigma[t] = sg;
      s_f[t] = irms / sg;
    }
#pragma unroll
    for (int i = 0; i < NVR; ++i) {
      const int i0 = 8 * (lane + 32 * i);
      const uint4 v = __ldg(xg + (static_cast<size_t>(t) * D + i0) / 8);
      uint4 o;
      o.x = bf16x2_to_f16x2_scaled(v.x, sg);
      o.y = bf16x2_to_f16x2_scaled(v.y, sg);
      o.z = bf16x2_to_f16x2_scaled(v.z, sg);
      o.w = bf16x2_to_f16x2_scaled(v.w, sg);
      if constexpr (TC) {
        // elements i0 + 2m, +1 (m = 0..3) are matrices (i0 % 32) / 2 + m of the segment
        uint8_t* b = reinterpret_cast<uint8_t*>(x16) + static_cast<size_t>(t) * XSTR + tc_b_offset(i0);
        *reinterpret_cast<uint32_t*>(b) = o.x;
        *reinterpret_cast<uint32_t*>(b + 16) = o.y;
        *reinterpret_cast<uint32_t*>(b + 32) = o.z;
        *reinterpret_cast<uint32_t*>(b + 48) = o.w;
      } else {
        *reinterpret_cast<uint4*>(x16 + static_cast<size_t>(t) * D + (((i0 & 31) >> 3) * (D / 32) + (i0 >> 5)) * 8) = o;
      }
    }
  }
  if constexpr (TC) {  // K-part sums and their arrival counts, used after the routing barrier
    for (int i = tid; i < p.tc_lt * 129; i += blockDim.x) tc_acc[i] = 0.f;
  }

  // gate/up of one staged chunk of `cu` units from unit uu, for the tokens
  // pair(i), i < nt (pair = token << 8 | slot); x is restaged in registers
  // only when the expert key or the token pass changes
  uint32_t xh[M::TGMAX * M::XS];
  int cur_key = -1, cur_g0 = -1;
  // pairs == nullptr: every token, slot kslot (the shared expert)
  auto compute_chunk = [&](const uint8_t* st, int cu, int uu, float sg, float su, int key, int nt,
                           const unsigned short* pairs, int kslot) {
    auto pair_of = [&](int i) { return pairs != nullptr ? static_cast<int>(pairs[i]) : ((i << 8) | kslot); };
    for (int g0 = 0; g0 < nt; g0 += M::TGMAX) {
      const int n = min(M::TGMAX, nt - g0);
      int hrow[M::TGMAX];
      float fg[M::TGMAX], fu[M::TGMAX];
#pragma unroll
      for (int t = 0; t < M::TGMAX; ++t) {
        const int pr = (t < n) ? pair_of(g0 + t) : 0;
        const int tok = pr >> 8;
        hrow[t] = tok * KS + (pr & 0xFF);
        fg[t] = (t < n) ? s_f[tok] * sg : 0.f;
        fu[t] = (t < n) ? s_f[tok] * su : 0.f;
      }
      if (key != cur_key || g0 != cur_g0) {
#pragma unroll
        for (int t = 0; t < M::TGMAX; ++t) {
          const int tok = pair_of(g0 + min(t, n - 1)) >> 8;
          const bool live = t < n;
#pragma unroll
          for (int xi = 0; xi < M::XV; ++xi) {
            const uint16_t* src = x16 + static_cast<size_t>(tok) * D + M::xblock(lane, xi) * 8;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 v = lds128(src + q * D / 4);  // chunk q of the block: q * (D/32) * 8 elements on
              xh[t * M::XS + xi * 16 + 4 * q + 0] = live ? v.x : 0u;
              xh[t * M::XS + xi * 16 + 4 * q + 1] = live ? v.y : 0u;
              xh[t * M::XS + xi * 16 + 4 * q + 2] = live ? v.z : 0u;
              xh[t * M::XS + xi * 16 + 4 * q + 3] = live ? v.w : 0u;
            }
          }
        }
        cur_key = key;
        cur_g0 = g0;
      }
      if (n == 1 && M::TGMAX > 1)
        gateup_chunk<D, 1>(st, cu, xh, lane, n, fg, fu, hrow, p.h, I, uu, p.htag, tag);
      else
        gateup_chunk<D, M::TGMAX>(st, cu, xh, lane, n, fg, fu, hrow, p.h, I, uu, p.htag, tag);
    }
  };

  // ---- P2: top-k (waits for every CTA's logits) and grouping, in every CTA
  // (called once by every warp, from inside the chunk loop below)
  auto routing_topk = [&]() {
    if (!ok && lane == 0) s_fail = 1;  // a wait of this warp gave up: the CTA stops together
    if (warp < T) {
      bool okt = false;
      if (ok) {
        const unsigned long long* lg = p.tlogits + (static_cast<size_t>(warp) * kLogitReplicas + c % kLogitReplicas) * E;
        if (E <= 256)
          okt = topk_warp_tagged<8>(lg, E, k, tag, &s_ids[warp * k], &s_gates[warp * k], lane, p.status);
        else
          okt = topk_warp_tagged<kMaxExperts / 32>(lg, E, k, tag, &s_ids[warp * k], &s_gates[warp * k], lane,
                                                   p.status);
      }
      if (!okt && lane == 0) s_fail = 1;
    }
    __syncthreads();
    if (s_fail) ok = false;
  };
  auto routing_group = [&]() {
    // the router rows are consumed by now (every warp's router tasks precede
    // this point), so their region serves as the grouping's scratch
    if (ok) cta_grouping(s_ids, T, k, E, S, dsc->act, dsc->off, dsc->pair, &dsc->n_routed, &dsc->n_active, rsm,
                         p.status);
    if (c == 0 && ok) {
      for (int i = tid; i < T * k; i += blockDim.x) {
        p.ids[i] = s_ids[i];
        p.gates[i] = s_gates[i];
        if (p.ids_out != nullptr) {
          p.ids_out[i] = s_ids[i];
          p.gates_out[i] = s_gates[i];
        }
      }
    }
  };

  // ---- P2 right after the router: top-k and grouping
  routing_topk();
  if (!ok) {
    drain_ring(bars, ns_g, consumed, issued, p.status);
    consumed = issued;
  }
  // One token: its k experts are distinct and each costs I units x 1 pass, so
  // the routed work split needs only their sorted ids, known right after the
  // top-k: the routed copies are issued before the grouping runs. Lane r of
  // every warp holds the r-th smallest id.
  const bool early = (!TC && T == 1) && ok;
  int my_act = 0, my_slot = 0;
  if (early) {
    const int v = lane < k ? s_ids[lane] : 0x7FFFFFFF;
    int rank = 0;
    for (int i = 0; i < k; ++i) rank += s_ids[i] < v ? 1 : 0;
    for (int j = 0; j < k; ++j) {
      const int vj = __shfl_sync(0xffffffffu, v, j), rj = __shfl_sync(0xffffffffu, rank, j);
      if (rj == lane) {
        my_act = vj;
        my_slot = j;
      }
    }
    // the grouping of one token: active slot a < k is the a-th smallest id,
    // serving the token once (pair = slot of that id in the top-k list); the
    // shared experts follow. Nothing reads the descriptor before the barrier
    // that ends the gate/up phase.
    if (warp == 0) {
      if (lane < k) {
        dsc->act[lane] = my_act;
        dsc->pair[lane] = static_cast<unsigned short>(my_slot);
      } else if (lane < k + S) {
        dsc->act[lane] = E + (lane - k);
        dsc->pair[lane] = static_cast<unsigned short>(lane);
      }
      if (lane <= k + S) dsc->off[lane] = lane;
      if (lane == 0) {
        dsc->n_routed = k;
        dsc->n_active = k + S;
      }
      if (c == 0 && lane < k) {
        p.ids[lane] = s_ids[lane];
        p.gates[lane] = s_gates[lane];
        if (p.ids_out != nullptr) {
          p.ids_out[lane] = s_ids[lane];
          p.gates_out[lane] = s_gates[lane];
        }
      }
    }
  }
  auto act_of = [&](int a) { return early ? __shfl_sync(0xffffffffu, my_act, a) : static_cast<int>(dsc->act[a]); };
  if (!early) routing_group();

  if constexpr (!TC) {
    // ---- P3: one stream of chunks per warp, issued and consumed in the same
    // order: phase 0 is this warp's slice of the shared expert's units (index =
    // unit; fetched since the start), phase 1 its range of the routed experts'
    // cost space (units x token passes; index = active expert * I + unit). One
    // loop, so the chunk code exists once.
    int u_begin = 0, u_end = 0;
    {
      const int n_routed = early ? k : (ok ? dsc->n_routed : 0);
      int* cost = s_cost[warp];
      if (!early) {
        cost_prefix(dsc, n_routed, I, M::TGMAX, cost, lane);
        __syncwarp();
      }
      // 32-bit arithmetic: C <= 65 experts x 1024 units x 4 passes and
      // gw < 240 * 16, so gw * C < 2^31
      const int C = early ? k * I : (n_routed > 0 ? cost[n_routed] : 0);
      // balance routed + shared work: warp w's routed range starts where the
      // combined cost w*(C + shared)/NW minus the shared cost of warps < w
      // falls (the shared units were split by warp index before the routing)
      const int ps = S > 0 ? (T + M::TGMAX - 1) / M::TGMAX : 0;  // passes of the shared expert
      const int CT = C + I * ps;
      auto rbound = [&](int w) { return min(C, max(0, w * CT / NW - (w * I / NW) * ps)); };
      // the bounds never decrease when each warp's share of CT covers the most
      // shared cost one warp can have
      const bool balanced = CT / NW >= ps * ((I + NW - 1) / NW);
      const int c_begin = balanced ? rbound(gw) : gw * C / NW;
      const int c_end = balanced ? (gw + 1 == NW ? C : rbound(gw + 1)) : (gw + 1) * C / NW;
      auto to_unit = [&](int cc, int& a, int& u) {
        int lo = 0, hi = n_routed - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (cost[mid] <= cc) lo = mid;
          else hi = mid - 1;
        }
        a = lo;
        const int passes = (dsc->off[a + 1] - dsc->off[a] + M::TGMAX - 1) / M::TGMAX;
        u = (cc - cost[a]) / passes;
      };
      if (early) {  // cost index == unit index (one pass per unit)
        u_begin = c_begin;
        u_end = c_end;
      } else if (c_end > c_begin) {
        int a0, u0, a1, u1;
        to_unit(c_begin, a0, u0);
        to_unit(c_end - 1, a1, u1);
        u_begin = a0 * I + u0;
        u_end = a1 * I + u1 + 1;
        if (c_begin > 0) {  // a unit already started by the previous warp's range is left to it
          int pa, pu;
          to_unit(c_begin - 1, pa, pu);
          if (pa == a0 && pu == u0) ++u_begin;
        }
      }
    }
    auto len_at = [&](int ph, int gg) {
      return ph == 0 ? min(M::CU, sh_end - gg) : min(M::CU, min(I - gg % I, u_end - gg));
    };
    auto settle = [&](int& ph, int& gg) {  // phase 0 exhausted -> start of phase 1
      if (ph == 0 && gg >= sh_end) {
        ph = 1;
        gg = u_begin;
      }
    };
    auto issue_at = [&](int ph, int gg) {
      const int e = ph == 0 ? E : act_of(gg / I);  // every lane (act_of may shuffle)
      if (lane == 0) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue_units(e, ph == 0 ? gg : gg % I, len_at(ph, gg), issued % ns_g);
      }
    };
    int iph = 0, ig = sh_issue;
    settle(iph, ig);
    while (ok && issued - consumed < ns_g && !(iph == 1 && ig >= u_end)) {
      issue_at(iph, ig);
      ig += len_at(iph, ig);
      settle(iph, ig);
      ++issued;
    }
    // then an L2 prefetch of this CTA's block of down rows of every routed
    // active expert (queued behind the gate/up copies)
    const int n_pf = early ? k : (ok ? dsc->n_routed : 0);
    for (int a = warp * 32 + lane; ok && a < n_pf && nrows > 0; a += kFusedWarps * 32) {
      const long long e = early ? my_act : dsc->act[a];  // early: a == lane
      prefetch_l2(p.codes + e * p.cpe + static_cast<long long>(I) * p.d + static_cast<long long>(n0) * ROWC,
                  nrows * ROWC);
      prefetch_l2(p.scales + e * p.spe + static_cast<long long>(I) * p.d / 8 + static_cast<long long>(n0) * ROWS,
                  nrows * ROWS);
    }
    {
      int cph = 0, cg = sh_begin, cur_a = -1;
      settle(cph, cg);
      float sg = S > 0 ? __ldg(p.tscale + 3 * E + 0) : 0.f, su = S > 0 ? __ldg(p.tscale + 3 * E + 1) : 0.f;
      while (ok && !(cph == 1 && cg >= u_end)) {
        const int cu = len_at(cph, cg);
        int key, nt, uu, kslot;
        const unsigned short* pairs;
        if (cph == 0) {
          key = -2;
          nt = T;
          uu = cg;
          pairs = nullptr;
          kslot = k;
        } else {
          const int a = cg / I;
          if (a != cur_a) {  // tensor scales of the expert, fetched before the stage wait
            const int e = act_of(a);
            sg = __ldg(p.tscale + 3 * e + 0);
            su = __ldg(p.tscale + 3 * e + 1);
            cur_a = a;
          }
          key = a;
          uu = cg % I;
          if (early) {  // one token, in the slot the lane-held ids give
            nt = 1;
            pairs = nullptr;
            kslot = __shfl_sync(0xffffffffu, my_slot, a);
          } else {
            const int pb = dsc->off[a];
            nt = dsc->off[a + 1] - pb;
            pairs = dsc->pair + pb;
            kslot = 0;
          }
        }
        const int slot = consumed % ns_g;
        if (!mbar_wait(&bars[slot], (consumed / ns_g) & 1, p.status)) {
          ok = false;
          break;
        }
        compute_chunk(ring + slot * p.stage_gateup, cu, uu, sg, su, key, nt, pairs, kslot);
        __syncwarp();
        ++consumed;
        cg += cu;
        settle(cph, cg);
        if (!(iph == 1 && ig >= u_end)) {
          issue_at(iph, ig);
          ig += len_at(iph, ig);
          settle(iph, ig);
          ++issued;
        }
      }
    }
  } else {
    // ---- P3, tensor-core variant: this CTA's local tiles are its shared
    // tiles, then a range of the routed experts' tiles, balanced against the
    // shared ones so every CTA gets about NT / G tiles
    const int n_routed = ok ? dsc->n_routed : 0;
    const int NR = n_routed * NTE, NT = NR + n_sh;
    // with NT >= G the balanced bounds never decrease (n_sh < G)
    const bool bal = NT >= G;
    auto rbound = [&](int cc) { return bal ? min(NR, max(0, cc * NT / G - cc * n_sh / G)) : cc * NR / G; };
    rt0 = rbound(c);
    const int rt1 = (c + 1 == G) ? NR : rbound(c + 1);
    const int L = nsh_c + rt1 - rt0;
    if (L > p.tc_lt) {  // the host sizes tc_lt above any split; never taken
      if (lane == 0) atomicOr(p.status, FLINT_DEVCHECK_MMA);
      ok = false;
    }
    const int n_items = (ok && L * KP > warp) ? (L * KP - 1 - warp) / kFusedWarps + 1 : 0;
    const int total = n_items * SPI;
    while (ok && issued - consumed < ns_g && issued < total) {
      if (lane == 0) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_issue(issued);
      }
      ++issued;
    }
    // then an L2 prefetch of this CTA's block of down rows of every routed
    // active expert (queued behind the gate/up copies)
    for (int a = warp * 32 + lane; ok && a < n_routed && nrows > 0; a += kFusedWarps * 32) {
      const long long e = dsc->act[a];
      prefetch_l2(p.codes + e * p.cpe + static_cast<long long>(I) * p.d + static_cast<long long>(n0) * ROWC,
                  nrows * ROWC);
      prefetch_l2(p.scales + e * p.spe + static_cast<long long>(I) * p.d / 8 + static_cast<long long>(n0) * ROWS,
                  nrows * ROWS);
    }
    const int g = lane >> 2, t = lane & 3;
    const int rg = 2 * tc_unit_of(g), ru = rg + 1;  // tile rows of MMA rows g (gate) and g + 8 (up)
    for (int m = 0; m < n_items && ok; ++m) {
      const int li = warp + kFusedWarps * m, lt = li / KP, part = li - lt * KP;
      int e, ti, a;
      tc_tile(lt, e, ti, a);
      const bool shared = a < 0;
      const int pb = shared ? 0 : dsc->off[a];
      const int n = shared ? T : dsc->off[a + 1] - pb;  // MMA columns in use (<= 8)
      auto pair_at = [&](int i) { return shared ? ((i << 8) | k) : static_cast<int>(dsc->pair[pb + i]); };
      // this lane's ldmatrix row: the token of column lane % 8 (unused columns repeat column 0)
      const uint8_t* xrow =
          reinterpret_cast<const uint8_t*>(x16) + static_cast<size_t>(pair_at((lane & 7) < n ? (lane & 7) : 0) >> 8) * XSTR;
      const float sg = __ldg(p.tscale + 3 * e + 0), su = __ldg(p.tscale + 3 * e + 1);
      float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
      for (int s = 0; s < SPI; ++s) {
        const int slot = consumed % ns_g;
        // warp-uniform outcome: the fragment loads and MMAs below need every lane
        if (!__all_sync(0xffffffffu, mbar_wait(&bars[slot], (consumed / ns_g) & 1, p.status))) {
          ok = false;
          break;
        }
        const uint8_t* cs = tc_codes + slot * kTcStageCodes;
        const uint8_t* ss = tc_scales + slot * kTcStageScales;
        const int seg0 = (part * SPI + s) * (kTcStageK / 128);
#pragma unroll 2
        for (int seg = 0; seg < kTcStageK / 128; ++seg) {
          uint32_t b[16];
          tc_load_b(xrow, (seg0 + seg) * 256, lane, b);
          const uint4 ca = lds128(tc_code_chunk(cs, rg, seg, t)), cb = lds128(tc_code_chunk(cs, ru, seg, t));
          const uint32_t sa = *reinterpret_cast<const uint16_t*>(ss + rg * 32 + seg * 8 + 2 * t);
          const uint32_t sb = *reinterpret_cast<const uint16_t*>(ss + ru * 32 + seg * 8 + 2 * t);
          tc_segment(acc, acc1, ca, cb, sa, sb, b);
        }
        __syncwarp();
        ++consumed;
        if (issued < total) {
          if (lane == 0) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc_issue(issued);
          }
          ++issued;
        }
      }
      if (!ok) break;
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[r] += acc1[r];
      // the tile's K parts meet in shared memory; the warp that arrives last
      // applies SwiGLU (two partial sums: their float sum is order-free)
      bool fin = true;
      if constexpr (KP > 1) {
        float* sl = tc_acc + static_cast<size_t>(lt) * 128;
#pragma unroll
        for (int r = 0; r < 4; ++r) atomicAdd(sl + r * 32 + lane, acc[r]);
        __syncwarp();
        int old = 0;
        if (lane == 0) {
          __threadfence_block();
          old = atomicAdd(tc_cnt + lt, 1);
        }
        old = __shfl_sync(0xffffffffu, old, 0);
        fin = old == KP - 1;
        if (fin) {
          __threadfence_block();
#pragma unroll
          for (int r = 0; r < 4; ++r) acc[r] = *reinterpret_cast<volatile const float*>(sl + r * 32 + lane);
        }
      }
      if (fin) {
        const int u = ti * kTcUnits + tc_unit_of(g);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int col = 2 * t + h2;
          if (col < n) {
            const int pr = pair_at(col), tok = pr >> 8;
            const float f = s_f[tok];
            const float hv = swiglu(acc[h2] * f * sg, acc[2 + h2] * f * su);
            st_tagged(p.htag + static_cast<size_t>(tok * KS + (pr & 0xFF)) * I + u, tag, hv);
          }
        }
      }
    }
  }
  if (!ok) drain_ring(bars, ns_g, consumed, issued, p.status);
  // every warp of this CTA is past its gate/up stages before the down phase
  // reuses their shared memory
  __syncthreads();
  const int n_active = ok ? dsc->n_active : 0;

  // ---- P4: down rows of this CTA's block of outputs, for every active expert
  // work area: [h16 R rows of HSTR bytes][s_y R x nb fp32][rings]; the
  // tensor-core variant lays it over everything after the descriptor (x16,
  // the router rows and the gate/up rings are dead by now)
  uint8_t* p4 = TC ? smem + ((sizeof(RouteDesc) + 127) & ~static_cast<size_t>(127)) : work;
  const size_t h16b = ((static_cast<size_t>(R) * HSTR) + 127) & ~static_cast<size_t>(127);
  uint16_t* h16 = reinterpret_cast<uint16_t*>(p4);
  float* s_y = reinterpret_cast<float*>(p4 + h16b);
  const size_t ybytes = ((sizeof(float) * static_cast<size_t>(R) * nb) + 127) & ~static_cast<size_t>(127);
  uint8_t* dring = p4 + h16b + ybytes + static_cast<size_t>(warp) * ns_d * p.stage_down;
  // the down ring uses this warp's barriers the gate/up ring left unused
  // (slots ns_g.. of its kMaxStages), so their phases start from zero
  uint64_t* bars_d = ring_bars + warp * kMaxStages + ns_g;
  const int RB = p.down_rb;
  const int nsub = (nrows + RB - 1) / RB;
  const int roff = RB * ROWC;
  const int n_items = (ok && nrows > 0) ? n_active * nsub : 0;
  int consumed_d = 0, issued_d = 0, next_issue = warp;
  auto issue_d = [&](int it, int slot) {
    const int a = it / nsub, sb = it % nsub;
    const int r0 = sb * RB, rows = min(RB, nrows - r0);
    const long long e = dsc->act[a];
    uint8_t* st = dring + slot * p.stage_down;
    mbar_arrive_expect_tx(&bars_d[slot], rows * (ROWC + ROWS));
    bulk_g2s(st, p.codes + e * p.cpe + static_cast<long long>(I) * p.d + static_cast<long long>(n0 + r0) * ROWC,
             rows * ROWC, &bars_d[slot]);
    bulk_g2s(st + roff, p.scales + e * p.spe + static_cast<long long>(I) * p.d / 8 + static_cast<long long>(n0 + r0) * ROWS,
             rows * ROWS, &bars_d[slot]);
  };
  // the rings overwrite smem last read through the generic proxy (gate/up
  // stages): order those reads before the bulk copies
  if (lane == 0) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  while (issued_d < ns_d && next_issue < n_items) {
    if (lane == 0) issue_d(next_issue, issued_d % ns_d);
    next_issue += kFusedWarps;
    ++issued_d;
  }
  // h rows (tagged, written by every CTA's gate/up) -> f16 rows with a
  // power-of-two scale each, converted once a row's I values all carry this
  // launch's tag: this wait is the layer's only cross-CTA dependency after the
  // routing. Element i of row P sits at P*I + ((i%32)/8 * VRD + i/32) * 8 + i%8,
  // so the 16-byte vectors the lanes of a down step read are contiguous.
  if (ok) {
    constexpr int F = I / 32;  // values per lane per row, element lane + 32*m
    // rows polled together per iteration (their L2 round trips overlap)
    constexpr int RPI = (TC && I <= 512) ? 2 : 1;
    constexpr unsigned kFull = (F >= 32) ? 0xFFFFFFFFu : ((1u << F) - 1u);
    for (int P0 = warp; P0 < R && ok; P0 += kFusedWarps * RPI) {
      float v[RPI][F];
      unsigned pend[RPI];
#pragma unroll
      for (int r = 0; r < RPI; ++r) pend[r] = (P0 + r * kFusedWarps < R) ? kFull : 0u;
      const long long t0 = clock64();
      for (;;) {
        unsigned long long w[RPI][F];
#pragma unroll
        for (int r = 0; r < RPI; ++r) {
          const unsigned long long* rowp = p.htag + static_cast<size_t>(P0 + r * kFusedWarps) * I;
#pragma unroll
          for (int m = 0; m < F; ++m) w[r][m] = (pend[r] & (1u << m)) ? ld_tagged(rowp + lane + 32 * m) : 0ull;
        }
        bool done = true;
#pragma unroll
        for (int r = 0; r < RPI; ++r) {
#pragma unroll
          for (int m = 0; m < F; ++m)
            if ((pend[r] & (1u << m)) && static_cast<uint32_t>(w[r][m] >> 32) == tag) {
              v[r][m] = __uint_as_float(static_cast<uint32_t>(w[r][m]));
              pend[r] &= ~(1u << m);
            }
          done = done && pend[r] == 0;
        }
        if (__all_sync(0xffffffffu, done)) break;
        if (clock64() - t0 > kWaitCycles) {
          ok = false;
          if (lane == 0) atomicOr(p.status, FLINT_DEVCHECK_WAIT);
          break;
        }
      }
      if (!ok) break;
#pragma unroll
      for (int r = 0; r < RPI; ++r) {
        const int P = P0 + r * kFusedWarps;
        if (P >= R) break;
        float amax = 0.f;
#pragma unroll
        for (int m = 0; m < F; ++m) amax = fmaxf(amax, fabsf(v[r][m]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float sig = pow2_scale_for(amax);
        if (lane == 0) s_hinv[P] = 1.f / sig;
#pragma unroll
        for (int m = 0; m < F; ++m) {
          const __half hv = __float2half_rn(v[r][m] * sig);
          const uint16_t hb = *reinterpret_cast<const uint16_t*>(&hv);
          if constexpr (TC)
            *reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(h16) + static_cast<size_t>(P) * HSTR +
                                         tc_b_offset(lane + 32 * m)) = hb;
          else
            h16[static_cast<size_t>(P) * I + (((lane >> 3) * VRD + m) << 3) + (lane & 7)] = hb;
        }
      }
    }
    if (!ok && lane == 0) s_fail = 1;
  }
  __syncthreads();
  if (s_fail) ok = false;
  // every CTA read this launch's generation before it wrote any h row, so the
  // generation can advance once all rows were seen
  if (c == 0 && tid == 0) asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p.counter + 1), "r"(gen + 1u) : "memory");
  const int rs = lane / VRD, cbk = lane % VRD;
  for (int it = warp; it < n_items && ok; it += kFusedWarps) {
    const int a = it / nsub, sb = it % nsub;
    const float sd = __ldg(p.tscale + 3 * dsc->act[a] + 2);
    const int slot = consumed_d % ns_d;
    if (!__all_sync(0xffffffffu, mbar_wait(&bars_d[slot], (consumed_d / ns_d) & 1, p.status))) {
      ok = false;
      break;
    }
    const uint8_t* st = dring + slot * p.stage_down;
    const int r0 = sb * RB, rows = min(RB, nrows - r0);
    if constexpr (TC) {
      // rows r0 + g and r0 + g + 8 of the block (MMA rows g, g + 8) against the
      // expert's h rows (columns); stage rows past `rows` hold stale bytes and
      // only reach discarded outputs
      const int pb = dsc->off[a], nt = dsc->off[a + 1] - pb;
      const int g = lane >> 2, t = lane & 3;
      auto hrow_at = [&](int i) {
        const int pr = dsc->pair[pb + i];
        return (pr >> 8) * KS + (pr & 0xFF);
      };
      const uint8_t* hb = reinterpret_cast<const uint8_t*>(h16) + static_cast<size_t>(hrow_at((lane & 7) < nt ? (lane & 7) : 0)) * HSTR;
      float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
      for (int seg = 0; seg < I / 128; ++seg) {
        uint32_t b[16];
        tc_load_b(hb, seg * 256, lane, b);
        const uint4 ca = lds128(st + g * ROWC + seg * 64 + t * 16);
        const uint4 cb = lds128(st + (g + 8) * ROWC + seg * 64 + t * 16);
        const uint32_t sa = *reinterpret_cast<const uint16_t*>(st + roff + g * ROWS + seg * 8 + 2 * t);
        const uint32_t sb = *reinterpret_cast<const uint16_t*>(st + roff + (g + 8) * ROWS + seg * 8 + 2 * t);
        tc_segment(acc, acc1, ca, cb, sa, sb, b);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) acc[r] += acc1[r];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int col = 2 * t + h2;
        if (col < nt) {
          const int P = hrow_at(col);
          const float ys = sd * s_hinv[P];
          if (g < rows) s_y[P * nb + r0 + g] = acc[h2] * ys;
          if (g + 8 < rows) s_y[P * nb + r0 + g + 8] = acc[2 + h2] * ys;
        }
      }
    } else {
      const int pb = dsc->off[a], nt = dsc->off[a + 1] - pb;
      for (int g0 = 0; g0 < nt; g0 += TGD) {
        const int n = min(TGD, nt - g0);
        uint32_t hh[TGD * 16];
        float yscale[TGD];
        int P[TGD];
  #pragma unroll
        for (int t = 0; t < TGD; ++t) {
          const int pr = dsc->pair[pb + g0 + min(t, n - 1)];
          P[t] = (pr >> 8) * KS + (pr & 0xFF);
          yscale[t] = sd * s_hinv[P[t]];
          const uint16_t* hp = h16 + static_cast<size_t>(P[t]) * I + cbk * 8;
  #pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 v = (t < n) ? lds128(hp + q * VRD * 8) : make_uint4(0u, 0u, 0u, 0u);
            hh[t * 16 + 4 * q + 0] = v.x;
            hh[t * 16 + 4 * q + 1] = v.y;
            hh[t * 16 + 4 * q + 2] = v.z;
            hh[t * 16 + 4 * q + 3] = v.w;
          }
        }
        // one pass: all rows of the block for these tokens, reduced once
        if (n == 1) {
          constexpr int V1 = 4;
          float o[V1 > VRD ? V1 / VRD : 1];
          down_block<I, 1>(st, roff, rows, hh, lane, o);
          if constexpr (V1 <= VRD) {
            const int rep = VRD / V1;  // lanes per value
            const int idx = cbk / rep, row = idx * RPS + rs;
            if (cbk % rep == 0 && row < rows) s_y[P[0] * nb + r0 + row] = o[0] * yscale[0];
          } else {
  #pragma unroll
            for (int g = 0; g < V1 / VRD; ++g) {
              const int idx = g * VRD + cbk, row = idx * RPS + rs;
              if (row < rows) s_y[P[0] * nb + r0 + row] = o[g] * yscale[0];
            }
          }
        } else {
          constexpr int VT = 4 * TGD;
          float o[VT > VRD ? VT / VRD : 1];
          down_block<I, TGD>(st, roff, rows, hh, lane, o);
          if constexpr (VT <= VRD) {
            const int rep = VRD / VT;
            const int idx = cbk / rep, step = idx / TGD, t = idx % TGD, row = step * RPS + rs;
            if (cbk % rep == 0 && t < n && row < rows) s_y[P[t] * nb + r0 + row] = o[0] * yscale[t];
          } else {
  #pragma unroll
            for (int g = 0; g < VT / VRD; ++g) {
              const int idx = g * VRD + cbk, step = idx / TGD, t = idx % TGD, row = step * RPS + rs;
              if (t < n && row < rows) s_y[P[t] * nb + r0 + row] = o[g] * yscale[t];
            }
          }
        }
      }
    }
    __syncwarp();
    ++consumed_d;
    if (next_issue < n_items) {
      if (lane == 0) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue_d(next_issue, issued_d % ns_d);
      }
      next_issue += kFusedWarps;
      ++issued_d;
    }
  }
  if (!ok) drain_ring(bars_d, ns_d, consumed_d, issued_d, p.status);
  __syncthreads();
  if (!ok) return;
  for (int idx = tid; idx < T * nrows; idx += blockDim.x) {
    const int t = idx / nrows, r = idx % nrows;
    float y = 0.f;
    for (int j = 0; j < k; ++j) y = fmaf(s_gates[t * k + j], s_y[(t * KS + j) * nb + r], y);
    for (int s = 0; s < S; ++s) y += s_y[(t * KS + k + s) * nb + r];
    const size_t o = static_cast<size_t>(t) * p.d + n0 + r;
    if (p.residual != nullptr) y += bf16_bits_to_f32(__ldcg(p.residual + o));
    const __nv_bfloat16 b = __float2bfloat16_rn(y);
    p.out[o] = *reinterpret_cast<const uint16_t*>(&b);
  }
}

}  // namespace flint
