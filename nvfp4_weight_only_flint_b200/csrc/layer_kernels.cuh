// layer_kernels.cuh -- the small-batch layer path, three kernels per layer
// chained with programmatic dependent launch:
//
//   k_route   Prologue (before waiting on the previous kernel): the router rows
//             and the shared expert's gate/up units are loaded into registers.
//             Then x is staged in shared memory by one bulk copy, per-token
//             scales are computed, router logits (warp per expert row) and the
//             shared expert's SwiGLU intermediates are produced. The last CTA to
//             finish runs top-k by warp shuffles and the token grouping, and
//             publishes a routing descriptor.
//   k_gateup  Bulk-copies the descriptor (and x) into shared memory, streams
//             the routed experts' gate/up units through per-warp bulk-copy
//             rings (chunks of consecutive units of one expert), dequantises in
//             registers, reduces with a transposed warp butterfly and writes
//             h = silu(g)*u. Warms L2 with the down rows of every active expert.
//   k_down    Bulk-copies the descriptor and every h row into shared memory,
//             streams (active expert, row block) items of down rows through
//             per-warp rings, and combines sum_j gate_j y_j + y_shared
//             (+ residual) in a fixed order for its block of output rows.
#pragma once

#include "gemv.cuh"

namespace flint {

constexpr int kRouteWarps = 8;
constexpr int kGemvWarps = 16;  // warps per CTA of the streaming kernels (<= 128 registers each)
constexpr int kDownTokens = 2;  // tokens per pass of the down kernel

// ----------------------------------------------------------------- warp-ring helpers
__device__ __forceinline__ void init_bars(uint64_t* bars, int n) {
  if (threadIdx.x == 0) {
    for (int i = 0; i < n; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
  }
}

// Every copy this warp started has landed (used on an aborted wait).
__device__ __forceinline__ void drain_ring(uint64_t* bars, int ns, int consumed, int issued, int* status) {
  for (int i = consumed; i < issued; ++i) mbar_wait(&bars[i % ns], (i / ns) & 1, status);
}

// ----------------------------------------------------------------- router only (any T)
// Warp per expert row and block of kRouterTokens tokens (grid.y), x read
// through L1. Used by flint_moe_route and the tensor-core path.
constexpr int kRouterTokens = 8;
template <int D>
__global__ void __launch_bounds__(256) k_router_only(LayerParams p) {
  constexpr int NVR = D / 256;
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (e >= p.E) return;
  uint4 wv[NVR];
  const uint4* row = reinterpret_cast<const uint4*>(p.wr + static_cast<size_t>(e) * D);
#pragma unroll
  for (int i = 0; i < NVR; ++i) wv[i] = __ldg(row + lane + 32 * i);
  const int t_end = min(p.T, static_cast<int>(blockIdx.y + 1) * kRouterTokens);
  for (int t = blockIdx.y * kRouterTokens; t < t_end; ++t) {
    const uint4* xr = reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(t) * D);
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < NVR; ++i) {
      const uint4 xv = __ldg(xr + lane + 32 * i);
      const uint32_t ww[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
      const uint32_t xx[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc = fmaf(bf16_bits_to_f32(ww[q] & 0xFFFFu), bf16_bits_to_f32(xx[q] & 0xFFFFu), acc);
        acc = fmaf(__uint_as_float(ww[q] & 0xFFFF0000u), __uint_as_float(xx[q] & 0xFFFF0000u), acc);
      }
    }
    acc = warp_sum(acc);
    if (lane == 0) p.logits[static_cast<size_t>(t) * p.E + e] = acc;
  }
}

__global__ void __launch_bounds__(256) k_topk(LayerParams p) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x * 8 + warp;
  if (t >= p.T) return;
  topk_token(p.logits + static_cast<size_t>(t) * p.E, p.E, p.k, p.ids + static_cast<size_t>(t) * p.k,
            p.gates + static_cast<size_t>(t) * p.k, lane);
}

// ----------------------------------------------------------------- k_route
template <int D>
__global__ void __launch_bounds__(kRouteWarps * 32, 1) k_route(LayerParams p) {
  using M = GateUpMap<D>;
  constexpr int NVR = D / 256;  // 8-element bf16 router vectors per lane
  extern __shared__ __align__(128) uint8_t smem[];  // x [T][D] bf16
  __shared__ float s_sigma[kMaxGemvTokens], s_irms[kMaxGemvTokens];
  __shared__ __align__(8) uint64_t s_bar;
  __shared__ int s_last;
  __shared__ Grouping g;
  __shared__ int s_ids[kMaxPairs];
  __shared__ float s_gates[kMaxPairs];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int task = blockIdx.x * kRouteWarps + warp;
  const int T = p.T, E = p.E, k = p.k;
  const int n_shared = p.S * p.I;
  const bool is_router = task < E;
  const bool is_shared = !is_router && task < E + n_shared;

  // Prologue: weights, which the preceding kernel in the stream does not write.
  uint4 wv[NVR];
  uint4 cv[M::NVU];
  uint32_t sv[M::NVU];
  float tsg = 0.f, tsu = 0.f;
  if (is_router) {
    const uint4* row = reinterpret_cast<const uint4*>(p.wr + static_cast<size_t>(task) * D);
#pragma unroll
    for (int i = 0; i < NVR; ++i) wv[i] = __ldg(row + lane + 32 * i);
  } else if (is_shared) {
    const int u = task - E;
    const uint8_t* cu = p.codes + static_cast<long long>(E) * p.cpe + static_cast<long long>(u) * D;
    const uint8_t* su = p.scales + static_cast<long long>(E) * p.spe + static_cast<long long>(u) * (D / 8);
#pragma unroll
    for (int j = 0; j < M::NVU; ++j) {
      int co, so, r, xi;
      M::vec(lane, j, co, so, r, xi);
      cv[j] = __ldg(reinterpret_cast<const uint4*>(cu + co));
      sv[j] = __ldg(reinterpret_cast<const uint16_t*>(su + so));
    }
    tsg = __ldg(p.tscale + 3 * E + 0);
    tsu = __ldg(p.tscale + 3 * E + 1);
  }
  if (tid == 0) {
    mbar_init(&s_bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();

  // x -> shared memory in one bulk copy.
  const uint32_t xbytes = static_cast<uint32_t>(T) * D * 2;
  if (tid == 0) {
    mbar_arrive_expect_tx(&s_bar, xbytes);
    bulk_g2s(smem, p.x, xbytes, &s_bar);
  }
  const bool x_ok = mbar_wait(&s_bar, 0, p.status);
  const uint16_t* xs = reinterpret_cast<const uint16_t*>(smem);

  // Per-token statistics, one warp per token.
  for (int t = warp; t < T && x_ok; t += kRouteWarps) {
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
    if (lane == 0) {
      s_sigma[t] = pow2_scale_for(amax);
      s_irms[t] = p.input_norm ? 1.f / sqrtf(ss / static_cast<float>(D) + kRmsEps) : 1.f;
    }
  }
  __syncthreads();

  if (is_router && x_ok) {
    for (int t = 0; t < T; ++t) {
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < NVR; ++i) {
        const uint4 xv = lds128(xs + static_cast<size_t>(t) * D + 8 * (lane + 32 * i));
        const uint32_t ww[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
        const uint32_t xx[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc = fmaf(bf16_bits_to_f32(ww[q] & 0xFFFFu), bf16_bits_to_f32(xx[q] & 0xFFFFu), acc);
          acc = fmaf(__uint_as_float(ww[q] & 0xFFFF0000u), __uint_as_float(xx[q] & 0xFFFF0000u), acc);
        }
      }
      acc = warp_sum(acc);
      if (lane == 0) p.logits[static_cast<size_t>(t) * E + task] = acc * s_irms[t];
    }
  } else if (is_shared && x_ok) {
    const int u = task - E;
    for (int t0 = 0; t0 < T; t0 += M::TGMAX) {
      const int n = min(M::TGMAX, T - t0);
      uint32_t xh[M::TGMAX * M::XS];
#pragma unroll
      for (int t = 0; t < M::TGMAX; ++t) {
#pragma unroll
        for (int xi = 0; xi < M::XV; ++xi) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 v = make_uint4(0, 0, 0, 0);
            float sg = 0.f;
            if (t < n) {
              v = lds128(xs + static_cast<size_t>(t0 + t) * D + 32 * M::xblock(lane, xi) + 8 * q);
              sg = s_sigma[t0 + t];
            }
            xh[t * M::XS + xi * 16 + 4 * q + 0] = bf16x2_to_f16x2_scaled(v.x, sg);
            xh[t * M::XS + xi * 16 + 4 * q + 1] = bf16x2_to_f16x2_scaled(v.y, sg);
            xh[t * M::XS + xi * 16 + 4 * q + 2] = bf16x2_to_f16x2_scaled(v.z, sg);
            xh[t * M::XS + xi * 16 + 4 * q + 3] = bf16x2_to_f16x2_scaled(v.w, sg);
          }
        }
      }
      float ag[M::TGMAX], au[M::TGMAX];
#pragma unroll
      for (int t = 0; t < M::TGMAX; ++t) ag[t] = au[t] = 0.f;
#pragma unroll
      for (int j = 0; j < M::NVU; ++j) {
        int co, so, r, xi;
        M::vec(lane, j, co, so, r, xi);
        float tmp[M::TGMAX];
#pragma unroll
        for (int t = 0; t < M::TGMAX; ++t) tmp[t] = 0.f;
        dot32_strided<M::TGMAX, M::XS>(cv[j], sv[j], xh + xi * 16, tmp);
#pragma unroll
        for (int t = 0; t < M::TGMAX; ++t) {
          ag[t] += r ? 0.f : tmp[t];
          au[t] += r ? tmp[t] : 0.f;
        }
      }
#pragma unroll
      for (int t = 0; t < M::TGMAX; ++t) {
        const float gs = warp_sum(ag[t]), us = warp_sum(au[t]);
        if (lane == 0 && t < n) {
          const int tok = t0 + t;
          const float f = s_irms[tok] / s_sigma[tok];
          const size_t P = static_cast<size_t>(tok) * (k + p.S) + k;
          p.h[P * p.I + u] = swiglu(gs * f * tsg, us * f * tsu);
        }
      }
    }
  }

  // Arrival; the last CTA routes and groups the tokens.
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    s_last = (atomicAdd(p.counter, 1u) == gridDim.x - 1) ? 1 : 0;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int t = warp; t < T; t += kRouteWarps)
    topk_token(p.logits + static_cast<size_t>(t) * E, E, k, &s_ids[t * k], &s_gates[t * k], lane);
  __syncthreads();
  for (int i = tid; i < T * k; i += blockDim.x) {
    p.ids[i] = s_ids[i];
    p.gates[i] = s_gates[i];
    if (p.ids_out != nullptr) {
      p.ids_out[i] = s_ids[i];
      p.gates_out[i] = s_gates[i];
    }
  }
  RouteDesc* d = p.desc;
  for (int t = tid; t < T; t += blockDim.x) {
    d->sigma[t] = s_sigma[t];
    d->irms[t] = s_irms[t];
  }
  if (T * k <= 64) {
    if (warp == 0) warp_grouping(s_ids, T, k, E, p.S, d, lane, p.status);
  } else {
    build_grouping(g, s_ids, T, k, E, p.S, p.status);
    if (tid == 0) {
      d->n_routed = g.n_routed;
      d->n_active = g.n_active;
    }
    for (int i = tid; i < g.n_active; i += blockDim.x) d->act[i] = g.act[i];
    for (int i = tid; i <= g.n_active; i += blockDim.x) d->off[i] = g.off[i];
    for (int i = tid; i < g.off[g.n_active]; i += blockDim.x) d->pair[i] = g.pair[i];
  }
  __syncthreads();
  __threadfence();
  if (tid == 0) atomicExch(p.counter, 0u);
}

// ----------------------------------------------------------------- k_gateup
// One chunk (cu <= CU consecutive units of one expert, staged at `st`) against
// TG tokens. Writes h for the chunk's (unit, token) pairs.
// With htag != nullptr, h is written as tagged 64-bit words (tag << 32 | h
// bits, one relaxed store each) instead of plain fp32.
template <int D, int TG>
__device__ __forceinline__ void gateup_chunk(const uint8_t* st, int cu, const uint32_t* xh, int lane,
                                             int n, const float* fscale_g, const float* fscale_u,
                                             const int* hrow, float* h, int I, int u0,
                                             unsigned long long* htag = nullptr, uint32_t tag = 0) {
  using M = GateUpMap<D>;
  constexpr int V = TG * 2;  // (token, gate|up) partial sums per unit
  constexpr int LV = ilog2(V);
  // one unit per iteration, reduced on its own: a rolled loop keeps the code
  // this runs (once or twice per launch at decode batch) small
#pragma unroll 1
  for (int c = 0; c < cu; ++c) {
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.f;
#pragma unroll
    for (int j = 0; j < M::NVU; ++j) {
      int co, so, r, xi;
      M::vec(lane, j, co, so, r, xi);
      const uint4 cvec = lds128(st + c * M::UNIT_CODE + co);
      const uint32_t s2 = *reinterpret_cast<const uint16_t*>(st + M::CU * M::UNIT_CODE + c * M::UNIT_SCALE + so);
      float tmp[TG];
#pragma unroll
      for (int t = 0; t < TG; ++t) tmp[t] = 0.f;
      dot32_strided<TG, M::XS>(cvec, s2, xh + xi * 16, tmp);
#pragma unroll
      for (int t = 0; t < TG; ++t) {
        if constexpr (M::VR >= 32) {
          acc[(t << 1) | (j / M::XV)] += tmp[t];
        } else {
          acc[t << 1] += r ? 0.f : tmp[t];
          acc[(t << 1) | 1] += r ? tmp[t] : 0.f;
        }
      }
    }
    const float total = xreduce<32, V>(acc, lane);
    const int rep = 5 - LV;  // lanes per value = 1 << rep
    const float other = __shfl_xor_sync(0xffffffffu, total, 1 << rep);
    const int idx = lane >> rep;
    const int r = idx & 1, t = idx >> 1;
    if (r == 0 && (lane & ((1 << rep) - 1)) == 0 && t < n) {
      const float hv = swiglu(total * fscale_g[t], other * fscale_u[t]);
      const size_t o = static_cast<size_t>(hrow[t]) * I + u0 + c;
      if (htag != nullptr)
        st_tagged(htag + o, tag, hv);
      else
        h[o] = hv;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kGemvWarps * 32, 1) k_gateup(LayerParams p) {
  using M = GateUpMap<D>;
  // dynamic shared memory: [descriptor][x (optional)][rings]
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float s_ts[2 * (kMaxExperts + 1)];
  __shared__ float s_f[kMaxGemvTokens];  // irms / sigma per token
  __shared__ __align__(8) uint64_t s_bar[kGemvWarps * kMaxStages + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ns = p.ns_gateup, I = p.I, T = p.T, KS = p.k + p.S;
  RouteDesc* dsc = reinterpret_cast<RouteDesc*>(smem);
  uint8_t* xsm = smem + sizeof(RouteDesc);
  const size_t xbytes = p.x_in_smem ? static_cast<size_t>(T) * D * 2 : 0;
  uint8_t* ring = smem + sizeof(RouteDesc) + xbytes + static_cast<size_t>(warp) * ns * p.stage_gateup;
  uint64_t* bars = s_bar + warp * ns;
  uint64_t* pbar = s_bar + kGemvWarps * kMaxStages;  // descriptor + x
  init_bars(s_bar, kGemvWarps * kMaxStages + 1);
  __syncthreads();
  pdl_wait();
  if (tid == 0) {
    mbar_arrive_expect_tx(pbar, static_cast<uint32_t>(sizeof(RouteDesc) + xbytes));
    bulk_g2s(dsc, p.desc, sizeof(RouteDesc), pbar);
    if (xbytes) bulk_g2s(xsm, p.x, static_cast<uint32_t>(xbytes), pbar);
  }
  bool ok = mbar_wait(pbar, 0, p.status);
  const int n_routed = dsc->n_routed, n_active = dsc->n_active;
  for (int i = tid; i < n_active; i += blockDim.x) {
    const int e = dsc->act[i];
    s_ts[2 * i] = __ldg(p.tscale + 3 * e + 0);
    s_ts[2 * i + 1] = __ldg(p.tscale + 3 * e + 1);
  }
  for (int t = tid; t < T; t += blockDim.x) s_f[t] = dsc->irms[t] / dsc->sigma[t];
  __syncthreads();
  pdl_trigger();

  // Warm L2 with this CTA's block of down rows of every active expert.
  if (tid < n_active && ok) {
    const int nb = p.down_nb, n0 = blockIdx.x * nb;
    if (n0 < p.d) {
      const int rows = min(nb, p.d - n0);
      const long long e = dsc->act[tid];
      prefetch_l2(p.codes + e * p.cpe + static_cast<long long>(I) * p.d + static_cast<long long>(n0) * (I / 2),
                  rows * (I / 2));
      prefetch_l2(p.scales + e * p.spe + static_cast<long long>(I) * p.d / 8 + static_cast<long long>(n0) * (I / 16),
                  rows * (I / 16));
    }
  }

  // This warp's contiguous range of routed (expert, unit) items, in chunks of
  // up to CU units of one expert.
  const long long NU = static_cast<long long>(n_routed) * I;
  const long long NW = static_cast<long long>(gridDim.x) * kGemvWarps;
  const long long gw = static_cast<long long>(blockIdx.x) * kGemvWarps + warp;
  const int u_begin = ok ? static_cast<int>(gw * NU / NW) : 0;
  const int u_end = ok ? static_cast<int>((gw + 1) * NU / NW) : 0;
  auto chunk_len = [&](int u) { return min(M::CU, min(I - u % I, u_end - u)); };
  int issue_u = u_begin, issued = 0;
  auto issue = [&](int u, int slot) {
    const int a = u / I, u0 = u % I, cu = chunk_len(u);
    const long long e = dsc->act[a];
    uint8_t* st = ring + slot * p.stage_gateup;
    mbar_arrive_expect_tx(&bars[slot], cu * M::UNIT_BYTES);
    bulk_g2s(st, p.codes + e * p.cpe + static_cast<long long>(u0) * D, cu * M::UNIT_CODE, &bars[slot]);
    bulk_g2s(st + M::CU * M::UNIT_CODE, p.scales + e * p.spe + static_cast<long long>(u0) * (D / 8),
             cu * M::UNIT_SCALE, &bars[slot]);
  };
  while (issued < ns && issue_u < u_end) {
    if (lane == 0) issue(issue_u, issued % ns);
    issue_u += chunk_len(issue_u);
    ++issued;
  }

  uint32_t xh[M::TGMAX * M::XS];
  int cur_a = -1, cur_g = -1;
  int consumed = 0;
  for (int u = u_begin; u < u_end;) {
    const int a = u / I, u0 = u % I, cu = chunk_len(u);
    const int slot = consumed % ns;
    if (!mbar_wait(&bars[slot], (consumed / ns) & 1, p.status)) {
      ok = false;
      break;
    }
    const uint8_t* st = ring + slot * p.stage_gateup;
    const int pb = dsc->off[a], nt = dsc->off[a + 1] - pb;
    const float sg = s_ts[2 * a], su = s_ts[2 * a + 1];
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
      if (a != cur_a || g0 != cur_g) {
#pragma unroll
        for (int t = 0; t < M::TGMAX; ++t) {
          const int tok = dsc->pair[pb + g0 + min(t, n - 1)] >> 8;
          const float sgm = (t < n) ? dsc->sigma[tok] : 0.f;
#pragma unroll
          for (int xi = 0; xi < M::XV; ++xi) {
            const size_t off = static_cast<size_t>(tok) * D + 32 * M::xblock(lane, xi);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 v = p.x_in_smem ? lds128(reinterpret_cast<const uint16_t*>(xsm) + off + 8 * q)
                                          : __ldcg(reinterpret_cast<const uint4*>(p.x + off) + q);
              xh[t * M::XS + xi * 16 + 4 * q + 0] = bf16x2_to_f16x2_scaled(v.x, sgm);
              xh[t * M::XS + xi * 16 + 4 * q + 1] = bf16x2_to_f16x2_scaled(v.y, sgm);
              xh[t * M::XS + xi * 16 + 4 * q + 2] = bf16x2_to_f16x2_scaled(v.z, sgm);
              xh[t * M::XS + xi * 16 + 4 * q + 3] = bf16x2_to_f16x2_scaled(v.w, sgm);
            }
          }
        }
        cur_a = a;
        cur_g = g0;
      }
      if (n == 1 && M::TGMAX > 1)
        gateup_chunk<D, 1>(st, cu, xh, lane, n, fg, fu, hrow, p.h, I, u0);
      else
        gateup_chunk<D, M::TGMAX>(st, cu, xh, lane, n, fg, fu, hrow, p.h, I, u0);
    }
    __syncwarp();
    ++consumed;
    u += cu;
    if (issue_u < u_end) {
      if (lane == 0) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue(issue_u, issued % ns);
      }
      issue_u += chunk_len(issue_u);
      ++issued;
    }
  }
  if (!ok) drain_ring(bars, ns, consumed, issued, p.status);
}

// ----------------------------------------------------------------- k_down
// A work item is (active expert, block of RB output rows); all of the expert's
// tokens are processed in passes of kDownTokens against the staged rows.
template <int I>
__global__ void __launch_bounds__(kGemvWarps * 32, 1) k_down(LayerParams p) {
  constexpr int VR = I / 32;    // 16-byte vectors per down row
  constexpr int RPS = 32 / VR;  // rows per warp step
  constexpr int TGD = kDownTokens;
  constexpr int ROWC = I / 2, ROWS = I / 16;
  // dynamic shared memory: [descriptor][h (optional)][s_y][rings]
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float s_gates[kMaxPairs];
  __shared__ float s_tsd[kMaxExperts + 1];
  __shared__ __align__(8) uint64_t s_bar[kGemvWarps * kMaxStages + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ns = p.ns_down, NB = p.down_nb, RB = p.down_rb, T = p.T, k = p.k, KS = p.k + p.S;
  const int n0 = blockIdx.x * NB;
  const int nrows = min(NB, p.d - n0);
  const int nsub = (nrows + RB - 1) / RB;
  RouteDesc* dsc = reinterpret_cast<RouteDesc*>(smem);
  const size_t hbytes = p.h_in_smem ? static_cast<size_t>(T) * KS * I * 4 : 0;
  float* hsm = reinterpret_cast<float*>(smem + sizeof(RouteDesc));
  float* s_y = reinterpret_cast<float*>(smem + sizeof(RouteDesc) + hbytes);
  const size_t ybytes = ((sizeof(float) * static_cast<size_t>(T) * KS * NB) + 127) & ~static_cast<size_t>(127);
  uint8_t* ring = smem + sizeof(RouteDesc) + hbytes + ybytes + static_cast<size_t>(warp) * ns * p.stage_down;
  uint64_t* bars = s_bar + warp * ns;
  uint64_t* pbar = s_bar + kGemvWarps * kMaxStages;
  const int roff = RB * ROWC;  // scales follow the codes in a stage
  init_bars(s_bar, kGemvWarps * kMaxStages + 1);
  __syncthreads();
  pdl_wait();
  if (tid == 0) {
    mbar_arrive_expect_tx(pbar, static_cast<uint32_t>(sizeof(RouteDesc) + hbytes));
    bulk_g2s(dsc, p.desc, sizeof(RouteDesc), pbar);
    if (hbytes) bulk_g2s(hsm, p.h, static_cast<uint32_t>(hbytes), pbar);
  }
  for (int i = tid; i < T * k; i += blockDim.x) s_gates[i] = __ldcg(p.gates + i);
  bool ok = mbar_wait(pbar, 0, p.status);
  const int n_active = dsc->n_active;
  for (int i = tid; i < n_active; i += blockDim.x) s_tsd[i] = __ldg(p.tscale + 3 * dsc->act[i] + 2);
  __syncthreads();
  pdl_trigger();

  const int n_items = ok ? n_active * nsub : 0;
  auto issue = [&](int it, int slot) {
    const int a = it / nsub, sb = it % nsub;
    const int r0 = sb * RB, rows = min(RB, nrows - r0);
    const long long e = dsc->act[a];
    uint8_t* st = ring + slot * p.stage_down;
    mbar_arrive_expect_tx(&bars[slot], rows * (ROWC + ROWS));
    bulk_g2s(st, p.codes + e * p.cpe + static_cast<long long>(I) * p.d + static_cast<long long>(n0 + r0) * ROWC,
             rows * ROWC, &bars[slot]);
    bulk_g2s(st + roff, p.scales + e * p.spe + static_cast<long long>(I) * p.d / 8 + static_cast<long long>(n0 + r0) * ROWS,
             rows * ROWS, &bars[slot]);
  };
  int issued = 0, next_issue = warp;
  while (issued < ns && next_issue < n_items) {
    if (lane == 0) issue(next_issue, issued % ns);
    next_issue += kGemvWarps;
    ++issued;
  }
  const int rs = lane / VR, cb = lane % VR;
  int consumed = 0;
  for (int it = warp; it < n_items; it += kGemvWarps) {
    const int slot = consumed % ns;
    if (!mbar_wait(&bars[slot], (consumed / ns) & 1, p.status)) {
      ok = false;
      break;
    }
    const uint8_t* st = ring + slot * p.stage_down;
    const int a = it / nsub, sb = it % nsub;
    const int r0 = sb * RB, rows = min(RB, nrows - r0);
    const int pb = dsc->off[a], nt = dsc->off[a + 1] - pb;
    const float sd = s_tsd[a];
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
            const float4 f = hbytes ? *reinterpret_cast<const float4*>(hsm + static_cast<size_t>(P[t]) * I + cb * 32 + 4 * q)
                                    : ldg_cg4(p.h + static_cast<size_t>(P[t]) * I + cb * 32 + 4 * q);
            v[4 * q] = f.x;
            v[4 * q + 1] = f.y;
            v[4 * q + 2] = f.z;
            v[4 * q + 3] = f.w;
          }
          float m = 0.f;
#pragma unroll
          for (int q = 0; q < 32; ++q) m = fmaxf(m, fabsf(v[q]));
          m = segment_max<VR>(m);
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
        const uint4 c = lds128(st + row * ROWC + cb * 16);
        const uint32_t s2 = *reinterpret_cast<const uint16_t*>(st + roff + row * ROWS + cb * 2);
        float acc[TGD];
#pragma unroll
        for (int t = 0; t < TGD; ++t) acc[t] = 0.f;
        if (n == 1)
          dot32_strided<1, 16>(c, s2, hh, acc);
        else
          dot32_strided<TGD, 16>(c, s2, hh, acc);
#pragma unroll
        for (int t = 0; t < TGD; ++t) {
          if (t < n) {
            const float y = segment_sum<VR>(acc[t]);
            if (cb == 0) s_y[P[t] * NB + r0 + row] = y * yscale[t];
          }
        }
      }
    }
    __syncwarp();
    ++consumed;
    if (next_issue < n_items) {
      if (lane == 0) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue(next_issue, issued % ns);
      }
      next_issue += kGemvWarps;
      ++issued;
    }
  }
  if (!ok) drain_ring(bars, ns, consumed, issued, p.status);
  __syncthreads();

  // Gated combine in a fixed order: routed slots 0..k-1, then the shared expert.
  for (int idx = tid; idx < T * nrows; idx += blockDim.x) {
    const int t = idx / nrows, r = idx % nrows;
    float y = 0.f;
    for (int j = 0; j < k; ++j) y = fmaf(s_gates[t * k + j], s_y[(t * KS + j) * NB + r], y);
    for (int s = 0; s < p.S; ++s) y += s_y[(t * KS + k + s) * NB + r];
    const size_t o = static_cast<size_t>(t) * p.d + n0 + r;
    if (p.residual != nullptr) y += bf16_bits_to_f32(__ldcg(p.residual + o));
    const __nv_bfloat16 b = __float2bfloat16_rn(y);
    p.out[o] = *reinterpret_cast<const uint16_t*>(&b);
  }
}

}  // namespace flint
