// fused_layer.cuh -- the whole layer in one persistent kernel (batch <= 8).
//
// One CTA per SM (8 warps), every SM busy in every phase:
//   P0  bulk copies of x and of this CTA's router rows; L2 prefetch of this
//       CTA's slice of the shared expert (gate/up units and down rows)
//   P1  router logits ((row, token) tasks over the warps) and per-token scales
//   --  grid barrier 1 (all logits written)
//   P2  every CTA: top-k of every token (sorted-list butterfly merge, warp per
//       token) and the token grouping (one warp), kept in shared memory
//   P3  gate/up of the routed experts and the shared expert through per-warp
//       bulk-copy rings, work split by compute cost; L2 prefetch of this CTA's
//       block of down rows of every routed active expert
//   --  grid barrier 2 (all h written)
//   P4  down: h staged in shared memory (or read from L2), down rows streamed
//       through per-warp rings, fixed-order gated combine (+ residual)
// The grid barrier is a flag per CTA in the workspace: a CTA publishes its epoch
// with a release store and polls every flag with relaxed loads (one round trip
// per poll, no atomics), then fences. Waits are bounded (FLINT_DEVCHECK_WAIT).
// The launch is cooperative, so every CTA is resident.
#pragma once

#include "layer_kernels.cuh"

namespace flint {

constexpr int kFusedMaxTokens = 8;
constexpr int kFusedWarps = 8;
constexpr int kMaxGridFlags = 240;  // CTAs of the persistent kernel (flags in the control block)

__device__ __forceinline__ unsigned ld_relaxed_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Grid barrier: this CTA stores `target` in its flag, then waits until every
// CTA's flag has reached `target` (wrap-safe comparison).
__device__ __forceinline__ bool flag_barrier(unsigned* flags, unsigned target, int* status, int* s_ok) {
  __syncthreads();
  if (threadIdx.x < 32) {
    if (threadIdx.x == 0)
      asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(flags + blockIdx.x), "r"(target) : "memory");
    const long long t0 = clock64();
    bool ok = true;
    for (;;) {
      bool mine = true;
      for (int i = threadIdx.x; i < static_cast<int>(gridDim.x); i += 32)
        mine &= static_cast<int>(ld_relaxed_u32(flags + i) - target) >= 0;
      if (__all_sync(0xffffffffu, mine)) break;
      if (clock64() - t0 > kWaitCycles) {
        ok = false;
        break;
      }
    }
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    if (threadIdx.x == 0) {
      *s_ok = ok ? 1 : 0;
      if (!ok) atomicOr(status, FLINT_DEVCHECK_WAIT);
    }
  }
  __syncthreads();
  return *s_ok != 0;
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

template <int D, int I>
__global__ void __launch_bounds__(kFusedWarps * 32, 1) k_layer(LayerParams p) {
  using M = GateUpMap<D>;
  constexpr int NVR = D / 256;   // router: 8-element bf16 vectors per lane
  constexpr int VRD = I / 32;    // down: 16-byte vectors per row
  constexpr int RPS = 32 / VRD;  // down: rows per warp step
  constexpr int TGD = kDownTokens;
  constexpr int ROWC = I / 2, ROWS = I / 16;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_ids[kFusedMaxTokens * kMaxTopK];
  __shared__ float s_gates[kFusedMaxTokens * kMaxTopK];
  __shared__ float s_sigma[kFusedMaxTokens], s_f[kFusedMaxTokens];
  __shared__ int s_cost[kFusedWarps][kFusedMaxTokens * kMaxTopK + 2];  // per-warp cost prefix over <= T*k+1 experts
  __shared__ unsigned s_base;
  __shared__ int s_ok;
  __shared__ __align__(8) uint64_t s_bar[kFusedWarps * kMaxStages + 3];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = p.T, E = p.E, k = p.k, S = p.S, KS = k + S, G = gridDim.x, c = blockIdx.x;
  unsigned* flags = p.counter + 15;  // control block bytes 64.. : one flag per CTA

  // ---- shared-memory carve-up: [desc][x][router rows][work]
  RouteDesc* dsc = reinterpret_cast<RouteDesc*>(smem);
  uint8_t* xsm = smem + sizeof(RouteDesc);
  const size_t xbytes = static_cast<size_t>(T) * D * 2;
  uint8_t* rsm = xsm + ((xbytes + 127) & ~static_cast<size_t>(127));
  const int rpc = (E + G - 1) / G;  // router rows per CTA
  uint8_t* work = rsm + static_cast<size_t>(rpc) * D * 2;
  uint64_t* ring_bars = s_bar;                          // [warp][kMaxStages]
  uint64_t* xbar = s_bar + kFusedWarps * kMaxStages;    // x
  uint64_t* rbar = xbar + 1;                            // router rows
  uint64_t* hbar = xbar + 2;                            // h staged for the down phase
  const int ns_g = p.ns_gateup, ns_d = p.ns_down;
  const int nb = p.down_nb, n0 = c * nb, nrows = max(0, min(nb, p.d - n0));
  const int r_begin = min(E, c * rpc), r_end = min(E, (c + 1) * rpc);

  // ---- P0: start the copies before anything else
  if (tid == 0) {
    for (int i = 0; i < kFusedWarps * kMaxStages + 3; ++i) mbar_init(&s_bar[i], 1);
    fence_barrier_init();
    mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(xbytes));
    bulk_g2s(xsm, p.x, static_cast<uint32_t>(xbytes), xbar);
    const uint32_t rbytes = static_cast<uint32_t>(r_end - r_begin) * D * 2;
    mbar_arrive_expect_tx(rbar, rbytes);
    if (rbytes) bulk_g2s(rsm, p.wr + static_cast<size_t>(r_begin) * D, rbytes, rbar);
    s_base = ld_relaxed_u32(flags + c);
  } else if (tid == 32 && S > 0) {
    const long long e = E;
    const int u0 = c * I / G, u1 = (c + 1) * I / G;
    if (u1 > u0) {
      prefetch_l2(p.codes + e * p.cpe + static_cast<long long>(u0) * D, (u1 - u0) * D);
      prefetch_l2(p.scales + e * p.spe + static_cast<long long>(u0) * (D / 8), (u1 - u0) * (D / 8));
    }
    if (nrows > 0) {
      prefetch_l2(p.codes + e * p.cpe + static_cast<long long>(I) * p.d + static_cast<long long>(n0) * ROWC, nrows * ROWC);
      prefetch_l2(p.scales + e * p.spe + static_cast<long long>(I) * p.d / 8 + static_cast<long long>(n0) * ROWS,
                  nrows * ROWS);
    }
  }
  __syncthreads();
  const unsigned base = s_base;

  // ---- P1: token statistics, router logits
  bool ok = mbar_wait(xbar, 0, p.status);
  const uint16_t* xs = reinterpret_cast<const uint16_t*>(xsm);
  float irms_t = 1.f;
  if (warp < T && ok) {
    const int t = warp;
    float amax = 0.f, ss = 0.f;
#pragma unroll
    for (int i = 0; i < NVR; ++i) {
      const uint4 v = lds128(xs + static_cast<size_t>(t) * D + 8 * (lane + 32 * i));
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
    irms_t = p.input_norm ? 1.f / sqrtf(ss / static_cast<float>(D) + kRmsEps) : 1.f;
    if (lane == 0) {
      const float sg = pow2_scale_for(amax);
      s_sigma[t] = sg;
      s_f[t] = irms_t / sg;
    }
  }
  __syncthreads();
  if (r_end > r_begin && ok) ok = mbar_wait(rbar, 0, p.status);
  for (int task = warp; task < (r_end - r_begin) * T && ok; task += kFusedWarps) {
    const int r = task / T, t = task % T;
    const uint16_t* wrow = reinterpret_cast<const uint16_t*>(rsm) + static_cast<size_t>(r) * D;
    float acc[NVR];
#pragma unroll
    for (int i = 0; i < NVR; ++i) {
      const uint4 wv = lds128(wrow + 8 * (lane + 32 * i));
      const uint4 xv = lds128(xs + static_cast<size_t>(t) * D + 8 * (lane + 32 * i));
      const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
      const uint32_t xx[4] = {xv.x, xv.y, xv.z, xv.w};
      float a = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a = fmaf(bf16_bits_to_f32(ww[q] & 0xFFFFu), bf16_bits_to_f32(xx[q] & 0xFFFFu), a);
        a = fmaf(__uint_as_float(ww[q] & 0xFFFF0000u), __uint_as_float(xx[q] & 0xFFFF0000u), a);
      }
      acc[i] = a;
    }
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < NVR; ++i) sum += acc[i];
    sum = warp_sum(sum);
    if (lane == 0) p.logits[static_cast<size_t>(t) * E + r_begin + r] = sum * s_f[t] * s_sigma[t];
  }
  if (!flag_barrier(flags, base + 1u, p.status, &s_ok)) ok = false;

  // ---- P2: top-k and grouping, in every CTA
  if (warp < T && ok)
    topk_token(p.logits + static_cast<size_t>(warp) * E, E, k, &s_ids[warp * k], &s_gates[warp * k], lane);
  __syncthreads();
  if (warp == 0 && ok) warp_grouping(s_ids, T, k, E, S, dsc, lane, p.status);
  __syncthreads();
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
  const int n_active = ok ? dsc->n_active : 0;
  // L2 prefetch of this CTA's block of down rows of every routed active expert
  if (tid < dsc->n_routed && nrows > 0 && ok) {
    const long long e = dsc->act[tid];
    prefetch_l2(p.codes + e * p.cpe + static_cast<long long>(I) * p.d + static_cast<long long>(n0) * ROWC, nrows * ROWC);
    prefetch_l2(p.scales + e * p.spe + static_cast<long long>(I) * p.d / 8 + static_cast<long long>(n0) * ROWS,
                nrows * ROWS);
  }

  // ---- P3: gate/up. This warp's range of the cost space, mapped to units.
  {
    int* cost = s_cost[warp];
    cost_prefix(dsc, n_active, I, M::TGMAX, cost, lane);
    __syncwarp();
    const long long C = n_active > 0 ? cost[n_active] : 0;
    const long long NW = static_cast<long long>(G) * kFusedWarps;
    const long long gw = static_cast<long long>(c) * kFusedWarps + warp;
    const long long c_begin = gw * C / NW, c_end = (gw + 1) * C / NW;
    auto to_unit = [&](long long cc, int& a, int& u) {
      int lo = 0, hi = n_active - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cost[mid] <= cc) lo = mid;
        else hi = mid - 1;
      }
      a = lo;
      const int passes = (dsc->off[a + 1] - dsc->off[a] + M::TGMAX - 1) / M::TGMAX;
      u = static_cast<int>((cc - cost[a]) / passes);
    };
    int g_begin = 0, g_end = 0;
    if (c_end > c_begin) {
      int a0, u0, a1, u1;
      to_unit(c_begin, a0, u0);
      to_unit(c_end - 1, a1, u1);
      g_begin = a0 * I + u0;
      g_end = a1 * I + u1 + 1;
      if (c_begin > 0) {  // a unit already started by the previous warp's range is left to it
        int pa, pu;
        to_unit(c_begin - 1, pa, pu);
        if (pa == a0 && pu == u0) ++g_begin;
      }
    }
    uint8_t* ring = work + static_cast<size_t>(warp) * ns_g * p.stage_gateup;
    uint64_t* bars = ring_bars + warp * kMaxStages;
    auto chunk_len = [&](int g) { return min(M::CU, min(I - g % I, g_end - g)); };
    auto issue = [&](int g, int slot) {
      const int a = g / I, uu = g % I, cu = chunk_len(g);
      const long long e = dsc->act[a];
      uint8_t* st = ring + slot * p.stage_gateup;
      mbar_arrive_expect_tx(&bars[slot], cu * M::UNIT_BYTES);
      bulk_g2s(st, p.codes + e * p.cpe + static_cast<long long>(uu) * D, cu * M::UNIT_CODE, &bars[slot]);
      bulk_g2s(st + M::CU * M::UNIT_CODE, p.scales + e * p.spe + static_cast<long long>(uu) * (D / 8),
               cu * M::UNIT_SCALE, &bars[slot]);
    };
    int issue_g = g_begin, issued = 0, consumed = 0;
    while (issued < ns_g && issue_g < g_end) {
      if (lane == 0) issue(issue_g, issued % ns_g);
      issue_g += chunk_len(issue_g);
      ++issued;
    }
    uint32_t xh[M::TGMAX * M::XS];
    int cur_a = -1, cur_g0 = -1;
    float sg = 0.f, su = 0.f;
    for (int g = g_begin; g < g_end;) {
      const int a = g / I, uu = g % I, cu = chunk_len(g);
      if (a != cur_a) {  // tensor scales of the expert, fetched before the stage wait
        const int e = dsc->act[a];
        sg = __ldg(p.tscale + 3 * e + 0);
        su = __ldg(p.tscale + 3 * e + 1);
      }
      const int slot = consumed % ns_g;
      if (!mbar_wait(&bars[slot], (consumed / ns_g) & 1, p.status)) {
        ok = false;
        break;
      }
      const uint8_t* st = ring + slot * p.stage_gateup;
      const int pb = dsc->off[a], nt = dsc->off[a + 1] - pb;
      for (int g0 = 0; g0 < nt; g0 += M::TGMAX) {
        const int n = min(M::TGMAX, nt - g0);
        int hrow[M::TGMAX];
        float fg[M::TGMAX], fu[M::TGMAX];
#pragma unroll
        for (int t = 0; t < M::TGMAX; ++t) {
          const int pr = (t < n) ? dsc->pair[pb + g0 + t] : 0;
          const int tok = pr >> 8;
          hrow[t] = tok * KS + (pr & 0xFF);
          fg[t] = (t < n) ? s_f[tok] * sg : 0.f;
          fu[t] = (t < n) ? s_f[tok] * su : 0.f;
        }
        if (a != cur_a || g0 != cur_g0) {
#pragma unroll
          for (int t = 0; t < M::TGMAX; ++t) {
            const int tok = dsc->pair[pb + g0 + min(t, n - 1)] >> 8;
            const float sgm = (t < n) ? s_sigma[tok] : 0.f;
#pragma unroll
            for (int xi = 0; xi < M::XV; ++xi) {
              const uint16_t* src = xs + static_cast<size_t>(tok) * D + 32 * M::xblock(lane, xi);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint4 v = lds128(src + 8 * q);
                xh[t * M::XS + xi * 16 + 4 * q + 0] = bf16x2_to_f16x2_scaled(v.x, sgm);
                xh[t * M::XS + xi * 16 + 4 * q + 1] = bf16x2_to_f16x2_scaled(v.y, sgm);
                xh[t * M::XS + xi * 16 + 4 * q + 2] = bf16x2_to_f16x2_scaled(v.z, sgm);
                xh[t * M::XS + xi * 16 + 4 * q + 3] = bf16x2_to_f16x2_scaled(v.w, sgm);
              }
            }
          }
          cur_g0 = g0;
        }
        cur_a = a;
        if (n == 1 && M::TGMAX > 1)
          gateup_chunk<D, 1>(st, cu, xh, lane, n, fg, fu, hrow, p.h, I, uu);
        else
          gateup_chunk<D, M::TGMAX>(st, cu, xh, lane, n, fg, fu, hrow, p.h, I, uu);
      }
      __syncwarp();
      ++consumed;
      g += cu;
      if (issue_g < g_end) {
        if (lane == 0) {
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          issue(issue_g, issued % ns_g);
        }
        issue_g += chunk_len(issue_g);
        ++issued;
      }
    }
    if (!ok) drain_ring(bars, ns_g, consumed, issued, p.status);
  }
  if (!flag_barrier(flags, base + 2u, p.status, &s_ok)) ok = false;

  // ---- P4: down rows of this CTA's block of outputs, for every active expert
  const size_t hbytes = p.h_in_smem ? static_cast<size_t>(T) * KS * I * 4 : 0;
  float* hsm = reinterpret_cast<float*>(work);
  float* s_y = reinterpret_cast<float*>(work + hbytes);
  const size_t ybytes = ((sizeof(float) * static_cast<size_t>(T) * KS * nb) + 127) & ~static_cast<size_t>(127);
  uint8_t* dring = work + hbytes + ybytes + static_cast<size_t>(warp) * ns_d * p.stage_down;
  // the down ring uses this warp's barriers the gate/up ring left unused
  // (slots ns_g.. of its kMaxStages), so their phases start from zero
  uint64_t* bars_d = ring_bars + warp * kMaxStages + ns_g;
  const int RB = p.down_rb;
  const int nsub = (nrows + RB - 1) / RB;
  const int roff = RB * ROWC;
  // the work area was last read through the generic proxy (gate/up stages);
  // order those reads before the bulk copies that overwrite it
  if (lane == 0) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (tid == 0 && hbytes && ok) {
    mbar_arrive_expect_tx(hbar, static_cast<uint32_t>(hbytes));
    bulk_g2s(hsm, p.h, static_cast<uint32_t>(hbytes), hbar);
  }
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
  while (issued_d < ns_d && next_issue < n_items) {
    if (lane == 0) issue_d(next_issue, issued_d % ns_d);
    next_issue += kFusedWarps;
    ++issued_d;
  }
  if (hbytes && ok) ok = mbar_wait(hbar, 0, p.status);
  const int rs = lane / VRD, cbk = lane % VRD;
  for (int it = warp; it < n_items && ok; it += kFusedWarps) {
    const int a = it / nsub, sb = it % nsub;
    const float sd = __ldg(p.tscale + 3 * dsc->act[a] + 2);
    const int slot = consumed_d % ns_d;
    if (!mbar_wait(&bars_d[slot], (consumed_d / ns_d) & 1, p.status)) {
      ok = false;
      break;
    }
    const uint8_t* st = dring + slot * p.stage_down;
    const int r0 = sb * RB, rows = min(RB, nrows - r0);
    const int pb = dsc->off[a], nt = dsc->off[a + 1] - pb;
    for (int g0 = 0; g0 < nt; g0 += TGD) {
      const int n = min(TGD, nt - g0);
      uint32_t hh[TGD * 16];
      float yscale[TGD];
      int P[TGD];
#pragma unroll
      for (int t = 0; t < TGD; ++t) {
        P[t] = 0;
        yscale[t] = 0.f;
        if (t < n) {
          const int pr = dsc->pair[pb + g0 + t];
          P[t] = (pr >> 8) * KS + (pr & 0xFF);
          float v[32];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 f = hbytes ? *reinterpret_cast<const float4*>(hsm + static_cast<size_t>(P[t]) * I + cbk * 32 + 4 * q)
                                    : ldg_cg4(p.h + static_cast<size_t>(P[t]) * I + cbk * 32 + 4 * q);
            v[4 * q] = f.x;
            v[4 * q + 1] = f.y;
            v[4 * q + 2] = f.z;
            v[4 * q + 3] = f.w;
          }
          float m = 0.f;
#pragma unroll
          for (int q = 0; q < 32; ++q) m = fmaxf(m, fabsf(v[q]));
          m = segment_max<VRD>(m);
          const float sig = pow2_scale_for(m);
          yscale[t] = sd / sig;
#pragma unroll
          for (int q = 0; q < 16; ++q) hh[t * 16 + q] = pack_f16x2(v[2 * q] * sig, v[2 * q + 1] * sig);
        } else {
#pragma unroll
          for (int q = 0; q < 16; ++q) hh[t * 16 + q] = 0u;
        }
      }
      for (int rr = 0; rr < rows; rr += RPS) {
        const int row = rr + rs;
        const uint4 cv = lds128(st + row * ROWC + cbk * 16);
        const uint32_t s2 = *reinterpret_cast<const uint16_t*>(st + roff + row * ROWS + cbk * 2);
        float acc[TGD];
#pragma unroll
        for (int t = 0; t < TGD; ++t) acc[t] = 0.f;
        if (n == 1)
          dot32_strided<1, 16>(cv, s2, hh, acc);
        else
          dot32_strided<TGD, 16>(cv, s2, hh, acc);
#pragma unroll
        for (int t = 0; t < TGD; ++t) {
          if (t < n) {
            const float y = segment_sum<VRD>(acc[t]);
            if (cbk == 0) s_y[P[t] * nb + r0 + row] = y * yscale[t];
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
