// tok1.cuh -- the layer at decode batch 1 as one cluster-per-expert kernel.
//
// The grid is (k + S) clusters of kTok1Cluster CTAs. Cluster j < k serves
// the expert the token routes to in top-k slot j; cluster k (when S = 1)
// serves the shared expert. Inside a cluster every exchange goes through
// distributed shared memory, so the only step that crosses clusters is the
// final gated sum, done by whichever CTA arrives last at a per-row-block
// counter (no CTA ever waits on another cluster):
//   P0  (before the dependency wait of programmatic dependent launch) bulk
//       copies of this CTA's slice of the router rows (routed clusters), or of
//       its slice of the shared expert (shared cluster): routing-independent
//   P1  the token's statistics, x staged as f16 in registers; this CTA's
//       router logits, written into every CTA of the cluster (DSMEM)
//   P2  cluster barrier; each CTA selects the top-k from its full copy of the
//       logits and issues one burst of bulk copies: its I/CS gate/up units and
//       its d/CS down rows of the cluster's expert
//   P3  gate/up + SwiGLU of its units as their copies land; each h value is
//       written into every CTA of the cluster (DSMEM); cluster barrier
//   P4  down rows of its block against the whole h, times the slot's gate:
//       fp32 partial sums of rows [rank*d/CS, (rank+1)*d/CS) of this slot
//   P5  the CTA that arrives last at its row block's counter adds the k + S
//       partials in slot order (+ residual), rounds to bf16 and resets it.
// The cluster barriers are hardware barriers that every CTA of a cluster
// reaches on every path; every mbarrier wait is bounded (FLINT_DEVCHECK_WAIT)
// and a CTA whose wait gave up still takes every later barrier and counter
// step, drains its copies and reports through the status word.
#pragma once

#include "gemv.cuh"

namespace flint {

constexpr int kTok1Cluster = 16;   // CTAs per cluster (non-portable size)
constexpr int kTok1Warps = 16;
constexpr int kTok1MaxChunks = 16;  // gate/up chunks (one per warp at most)
constexpr int kTok1ChunksPerCopy = 1;  // gate/up chunks one bulk copy (and its barrier) covers

struct Tok1Params {
  const uint16_t* x;         // [1][d] bf16
  const uint16_t* wr;        // [E][d] bf16
  const uint8_t* codes;      // packed E2M1 codes
  const uint8_t* scales;     // packed E4M3 block scales
  const float* tscale;       // [E+S][3]
  const uint16_t* residual;  // [1][d] bf16 or null
  uint16_t* out;             // [1][d] bf16
  int* status;               // workspace status word
  unsigned* rb_count;        // [kTok1Cluster] arrival counters per row block (workspace, zero between launches)
  float* partial;            // [k+S][d] gated fp32 partial outputs per slot (workspace)
  int* ids;                  // [k] routed ids (workspace)
  float* gates;              // [k]
  int* ids_out;              // optional public copies
  float* gates_out;
  long long cpe, spe;        // code / scale bytes per expert
  int E, k, S;
  int input_norm;
  int trigger_early;         // 1: allow the next kernel to launch at once
};

// Dynamic shared-memory bytes of k_tok1: the larger of the router-row slice and
// the expert slice (they share the region), then the cluster's logits, h
// (fp32, lane-interleaved: unit u at (u % 32) * (I/32) + u / 32), the token's
// x (bf16) and x as f16 in the lane-interleaved order (8-element chunk q of
// 32-element vector v at q * (d/32) + v), so that the lanes of a warp read
// consecutive words or 16-byte chunks.
__host__ __device__ constexpr size_t tok1_region_bytes(int D, int I, int E) {
  const size_t rows = static_cast<size_t>((E + kTok1Cluster - 1) / kTok1Cluster) * D * 2;
  const size_t ex = static_cast<size_t>(I / kTok1Cluster) * (D + D / 8) +
                    static_cast<size_t>(D / kTok1Cluster) * (I / 2 + I / 16);
  return ((rows > ex ? rows : ex) + 127) & ~static_cast<size_t>(127);
}
__host__ __device__ constexpr size_t tok1_smem_bytes(int D, int I, int E) {
  return tok1_region_bytes(D, I, E) + ((static_cast<size_t>(E) * 4 + 127) & ~static_cast<size_t>(127)) +
         static_cast<size_t>(I) * 4 + static_cast<size_t>(D) * 4;
}

__device__ __forceinline__ unsigned cluster_rank() {
  unsigned r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ unsigned cluster_index() {
  unsigned r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Named CTA barriers (id > 0) over `threads` threads, whole warps.
__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
__device__ __forceinline__ void named_arrive(int id, int threads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Store v into the same shared-memory variable of CTA `rank` of this cluster.
__device__ __forceinline__ void st_cluster_f32(float* local, unsigned rank, float v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(local)), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(v) : "memory");
}

__device__ __forceinline__ void st_cluster_u32(unsigned* local, unsigned rank, unsigned v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_addr(local)), "r"(rank));
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(remote), "r"(v) : "memory");
}

// Top-k of one token's E <= 32*NE logits by one warp, in k rolled rounds
// (every phase of this kernel runs once per launch, so its code size, not its
// loop overhead, is what costs: an unrolled sorting network would be fetched
// from L2 at every launch). Lane l holds the order-preserving codes of
// experts l + 32 i (0 = absent). A round takes each lane's best (largest code,
// the lowest i on ties), the warp maximum of those with redux.sync, then among
// the lanes holding it the lowest expert index (a second redux over
// 0xFFFFFFFF - e); the owner clears it. Ties go to the lower expert index,
// -0 equals +0 (route_code). Gates: exp(l_j - l_max) / sum over the selected.
template <int NE>
__device__ __forceinline__ void topk_rounds(uint32_t (&code)[NE], int k, int* ids, float* gates, int lane) {
  float my_val = 0.f, v0 = 0.f;
  int my_sel = 0;
  // slots already selected, as a bit mask: the code array is only read, so it
  // stays in registers (clearing a slot by a computed index had put it in
  // local memory)
  uint32_t taken = 0u;
#pragma unroll 1
  for (int r = 0; r < k; ++r) {
    uint32_t best = 0u;
    int bi = 0;
#pragma unroll
    for (int i = 0; i < NE; ++i) {
      const uint32_t c = ((taken >> i) & 1u) ? 0u : code[i];
      if (c > best) {
        best = c;
        bi = i;
      }
    }
    const uint32_t m = __reduce_max_sync(0xffffffffu, best);
    const uint32_t w = __reduce_max_sync(0xffffffffu, best == m ? 0xFFFFFFFFu - static_cast<uint32_t>(lane + 32 * bi) : 0u);
    const int e = static_cast<int>(0xFFFFFFFFu - w);
    if ((e & 31) == lane) taken |= 1u << (e >> 5);
    const float v = route_code_value(m);
    if (r == 0) v0 = v;
    if (lane == r) {
      my_val = v;
      my_sel = e;
    }
  }
  const float ex = (lane < k) ? __expf(my_val - v0) : 0.f;
  const float sum = warp_sum(ex);
  if (lane < k) {
    ids[lane] = my_sel;
    gates[lane] = ex * (1.f / sum);
  }
}

// NE: logit slots per lane of the top-k (E <= 32 * NE), 8 or 16.
template <int D, int I, int NE>
__global__ void __launch_bounds__(kTok1Warps * 32, 1) k_tok1(Tok1Params p) {
  constexpr int CS = kTok1Cluster;
  constexpr int VPR = D / 32;                     // 16-byte code vectors per gate/up row
  constexpr int XV = VPR >= 32 ? VPR / 32 : 1;    // x vectors (32 elements) per lane
  constexpr int UV = 2 * VPR / 32 > 0 ? 2 * VPR / 32 : 1;  // code vectors per lane per unit
  constexpr int UPC = I / CS;                     // gate/up units per CTA
  constexpr int CU = UPC >= kTok1Warps ? UPC / kTok1Warps : 1;  // units per chunk
  constexpr int NCH = UPC / CU;                   // chunks (<= 16)
  constexpr int RPC = D / CS;                     // down rows per CTA
  constexpr int LPR = I / 32;                     // lanes per down row (one 16-byte vector each)
  constexpr int RPS = 32 / LPR;                   // down rows per warp step
  constexpr int UNIT_C = D, UNIT_S = D / 8;       // bytes of a unit's codes / scales
  constexpr int DROW_C = I / 2, DROW_S = I / 16;  // bytes of a down row's codes / scales
  constexpr int CPC = kTok1ChunksPerCopy < NCH ? kTok1ChunksPerCopy : NCH;  // chunks per copy
  constexpr int NCP = NCH / CPC;                  // gate/up copies
  static_assert(NCH <= kTok1MaxChunks && NCH * CU == UPC && NCP * CPC == NCH, "chunking");
  static_assert(RPC % RPS == 0 || RPC < RPS, "down rows");

  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t s_bar[kTok1MaxChunks + 3];  // chunks, down rows, router rows, x
  __shared__ int s_ids[kMaxTopK];
  __shared__ float s_gates[kMaxTopK];
  __shared__ int s_fail, s_last, s_burst, s_expert;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = p.E, k = p.k, KS = k + p.S;
  const unsigned rank = cluster_rank();
  const int slot = static_cast<int>(cluster_index());  // top-k slot served, or k = shared
  const bool shared = slot >= k;
  uint8_t* region = smem;
  float* s_logits = reinterpret_cast<float*>(smem + tok1_region_bytes(D, I, E));
  float* s_h = s_logits + ((E + 31) & ~31);
  const uint16_t* s_x = reinterpret_cast<const uint16_t*>(s_h + I);
  uint16_t* x16 = const_cast<uint16_t*>(s_x) + D;  // f16, lane-interleaved
  uint8_t* gu_codes = region;                                   // [UPC][D]
  uint8_t* gu_scales = region + UPC * UNIT_C;                   // [UPC][D/8]
  uint8_t* dn_codes = gu_scales + UPC * UNIT_S;                 // [RPC][I/2]
  uint8_t* dn_scales = dn_codes + RPC * DROW_C;                 // [RPC][I/16]
  uint64_t* bar_chunk = s_bar;
  uint64_t* bar_down = s_bar + kTok1MaxChunks;
  uint64_t* bar_rows = s_bar + kTok1MaxChunks + 1;
  uint64_t* bar_x = s_bar + kTok1MaxChunks + 2;
  const int r0 = static_cast<int>(rank) * E / CS, r1 = (static_cast<int>(rank) + 1) * E / CS;

  // This CTA's slice of expert e: one copy per chunk and one for the down
  // rows, each from a lane of its own; `codes` selects the code copies (warp
  // 0) or the scale copies (warp 1), so that the two go out in parallel (a
  // thread takes ~0.25 us per bulk-copy operation). The barriers' byte counts
  // are set in P0: they do not depend on the routing.
  auto issue_expert = [&](int e, bool codes) {
    const uint8_t* cb = p.codes + static_cast<long long>(e) * p.cpe;
    const uint8_t* sb = p.scales + static_cast<long long>(e) * p.spe;
    const int u0 = static_cast<int>(rank) * UPC;
    constexpr int CCU = CPC * CU;  // units of one copy
    if (lane < NCP) {
      const int u = u0 + lane * CCU;
      if (codes)
        bulk_g2s(gu_codes + lane * CCU * UNIT_C, cb + static_cast<long long>(u) * UNIT_C, CCU * UNIT_C, &bar_chunk[lane]);
      else
        bulk_g2s(gu_scales + lane * CCU * UNIT_S, sb + static_cast<long long>(u) * UNIT_S, CCU * UNIT_S,
                 &bar_chunk[lane]);
    } else if (lane == NCP) {
      const long long n0 = static_cast<long long>(rank) * RPC;
      if (codes)
        bulk_g2s(dn_codes, cb + static_cast<long long>(I) * D + n0 * DROW_C, RPC * DROW_C, bar_down);
      else
        bulk_g2s(dn_scales, sb + static_cast<long long>(I) * D / 8 + n0 * DROW_S, RPC * DROW_S, bar_down);
    }
  };

  // ---- P0: routing-independent copies, before the dependency wait
  if (tid == 0) {
    for (int i = 0; i < kTok1MaxChunks + 3; ++i) mbar_init(&s_bar[i], 1);
    fence_barrier_init();
    s_fail = 0;
    s_burst = shared ? 1 : 0;
    if (!shared) {
      const uint32_t rbytes = static_cast<uint32_t>(r1 - r0) * D * 2;
      mbar_arrive_expect_tx(bar_rows, rbytes);
      if (rbytes) bulk_g2s(region, p.wr + static_cast<size_t>(r0) * D, rbytes, bar_rows);
    }
  }
  __syncthreads();
  if (warp == 0) {  // byte counts of the expert slice's barriers
    constexpr int CCU = CPC * CU;
    if (lane < NCP) mbar_arrive_expect_tx(&bar_chunk[lane], CCU * (UNIT_C + UNIT_S));
    else if (lane == NCP) mbar_arrive_expect_tx(bar_down, RPC * (DROW_C + DROW_S));
    else if (lane == NCP + 1) mbar_arrive_expect_tx(bar_x, D * 2);
  }
  if (shared && warp < 2) {  // the shared expert's slice needs no routing
    named_sync(1, 64);  // after the byte counts
    issue_expert(E, warp == 0);
  }
  // every CTA of the cluster must be running before any writes into its
  // shared memory: arrive now, wait just before the first remote store
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  if (p.trigger_early) pdl_trigger();
  pdl_wait();  // x (and the workspace) are written by the preceding kernel
  // one copy of x per CTA: every warp reading it from L2 would make its 32
  // lines a hot spot of thousands of requests
  if (tid == 0) bulk_g2s(const_cast<uint16_t*>(s_x), p.x, D * 2, bar_x);

  // ---- P1: every warp derives the token's statistics from the bf16 copy of
  // x (16-byte lanes, conflict-free; the same values in every warp, so no
  // barrier); warp w computes router rows r0 + w, r0 + w + 16, ... and stores
  // each logit into every CTA of the cluster; x is converted once into a
  // lane-interleaved f16 copy, from which each lane loads its x vectors
  // v = lane + 32 j (j < XV) of a gate/up row (at D = 512 lanes 16..31 repeat
  // lanes 0..15).
  bool ok = __all_sync(0xffffffffu, mbar_wait(bar_x, 0, p.status));
  if (!shared && r1 > r0 && !__all_sync(0xffffffffu, mbar_wait(bar_rows, 0, p.status))) ok = false;
  float sigma, irms;
  {
    float amax = 0.f, ss = 0.f;
    for (int i = lane; i < D / 8; i += 32) {
      const uint4 v = lds128(s_x + 8 * i);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float a = bf16_bits_to_f32(w4[q] & 0xFFFFu), b = __uint_as_float(w4[q] & 0xFFFF0000u);
        amax = fmaxf(amax, fmaxf(fabsf(a), fabsf(b)));
        ss = fmaf(a, a, ss);
        ss = fmaf(b, b, ss);
      }
    }
    amax = segment_max<32>(amax);
    ss = warp_sum(ss);
    sigma = pow2_scale_for(amax);
    irms = p.input_norm ? 1.f / sqrtf(ss / static_cast<float>(D) + kRmsEps) : 1.f;
  }
  const float fx = irms / sigma;  // dot(q, x*sigma) * fx = dot(q, x) * irms
  // every CTA of the cluster must be running before the remote stores: the
  // cluster arrival of P0 is waited for here
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  if (!shared && ok) {
    for (int r = r0 + warp; r < r1; r += kTok1Warps) {
      const uint8_t* row = region + static_cast<size_t>(r - r0) * D * 2;
      float a = 0.f;
#pragma unroll 4
      for (int i = lane; i < D / 8; i += 32) {
        const uint4 wv = lds128(row + 16 * i), xv = lds128(s_x + 8 * i);
        fma2_bf16_f32(wv.x, xv.x, a);
        fma2_bf16_f32(wv.y, xv.y, a);
        fma2_bf16_f32(wv.z, xv.z, a);
        fma2_bf16_f32(wv.w, xv.w, a);
      }
      const float logit = warp_sum(a) * irms;
      if (lane < CS) st_cluster_f32(s_logits + r, static_cast<unsigned>(lane), logit);
    }
  }
  for (int i = tid; i < D / 8; i += blockDim.x) {
    const uint4 v = lds128(s_x + 8 * i);
    uint4 o;
    o.x = bf16x2_to_f16x2_scaled(v.x, sigma);
    o.y = bf16x2_to_f16x2_scaled(v.y, sigma);
    o.z = bf16x2_to_f16x2_scaled(v.z, sigma);
    o.w = bf16x2_to_f16x2_scaled(v.w, sigma);
    *reinterpret_cast<uint4*>(x16 + (((i & 3) * VPR) + (i >> 2)) * 8) = o;  // vector i/4, chunk i%4
  }
  if (!ok && lane == 0) s_fail = 1;
  __syncthreads();
  const int xl = lane % VPR;  // first x vector of this lane
  uint32_t xr[XV][16];
#pragma unroll
  for (int j = 0; j < XV; ++j)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 v = lds128(x16 + ((q * VPR) + xl + 32 * j) * 8);
      xr[j][4 * q + 0] = v.x;
      xr[j][4 * q + 1] = v.y;
      xr[j][4 * q + 2] = v.z;
      xr[j][4 * q + 3] = v.w;
    }

  // ---- P2: every CTA of the cluster holds all E logits; select, then issue
  cluster_sync_all();
  if (s_fail) ok = false;
  if (!shared && warp == 0) {
    int e = -1;
    if (ok) {
      uint32_t code[NE];
#pragma unroll
      for (int i = 0; i < NE; ++i) {
        const int ei = lane + 32 * i;
        code[i] = (ei < E) ? max(route_code(s_logits[ei]), 1u) : 0u;
      }
      topk_rounds<NE>(code, k, s_ids, s_gates, lane);
      __syncwarp();
      e = s_ids[slot];
      if (e < 0 || e >= E) {
        if (lane == 0) atomicOr(p.status, FLINT_DEVCHECK_EXPERT_ID);
        e = -1;
      }
    }
    if (lane == 0) {
      s_expert = e;
      s_burst = e >= 0 ? 1 : 0;
    }
    // the router rows were read before the cluster barrier; order those
    // generic reads before the copies that overwrite them
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    named_arrive(1, 64);  // warp 1 takes the scale copies
    if (e >= 0) issue_expert(e, true);
    if (ok && slot == 0 && rank == 0 && lane < k) {
      p.ids[lane] = s_ids[lane];
      p.gates[lane] = s_gates[lane];
      if (p.ids_out != nullptr) {
        p.ids_out[lane] = s_ids[lane];
        p.gates_out[lane] = s_gates[lane];
      }
    }
  } else if (!shared && warp == 1) {
    named_sync(1, 64);
    const int e = s_expert;
    if (e >= 0) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue_expert(e, false);
    }
  }
  __syncthreads();
  const bool issued = s_burst != 0;  // this CTA's slice of an expert is on its way
  const int expert = shared ? E : (issued ? s_ids[slot] : 0);
  const float gate = shared ? 1.f : s_gates[slot];
  float sg = 0.f, su = 0.f, sd = 0.f;
  if (issued) {
    sg = __ldg(p.tscale + 3 * expert + 0);
    su = __ldg(p.tscale + 3 * expert + 1);
    sd = __ldg(p.tscale + 3 * expert + 2);
  }

  // ---- P3: gate/up of chunk `warp` (CU units), h into every CTA of the cluster
  bool ok3 = issued;
  if (warp < NCH && issued) {
    if (!__all_sync(0xffffffffu, mbar_wait(&bar_chunk[warp / CPC], 0, p.status))) ok3 = false;
    if (ok3) {
#pragma unroll 1
      for (int c = 0; c < CU; ++c) {
        const int ul = warp * CU + c;
        const uint8_t* uc = gu_codes + ul * UNIT_C;
        const uint8_t* us = gu_scales + ul * UNIT_S;
        float g = 0.f, u = 0.f;
#pragma unroll
        for (int j = 0; j < UV; ++j) {
          const int v = lane + 32 * j;  // vector of the unit (gate row: v < VPR)
          const uint4 cv = lds128(uc + 16 * v);
          const uint32_t s2 = *reinterpret_cast<const uint16_t*>(us + 2 * v);
          float acc = 0.f;
          dot32_strided<1, 16>(cv, s2, xr[VPR >= 32 ? j % XV : 0], &acc);
          if (v < VPR) g += acc;
          else u += acc;
        }
        g = warp_sum(g);
        u = warp_sum(u);
        const float hv = swiglu(g * fx * sg, u * fx * su);
        // stored lane-interleaved: unit u at (u % 32) * (I / 32) + u / 32, so
        // that the lanes of a down step read consecutive words
        const int uu = static_cast<int>(rank) * UPC + ul;
        if (lane < CS) st_cluster_f32(s_h + (uu & 31) * LPR + (uu >> 5), static_cast<unsigned>(lane), hv);
      }
    }
  }
  if (!ok3 && issued && lane == 0) s_fail = 1;
  cluster_sync_all();
  if (s_fail) ok = false;
  ok = ok && issued;

  // ---- P4: down rows of this CTA's block against the whole h
  float* part = p.partial + static_cast<size_t>(slot) * D + static_cast<size_t>(rank) * RPC;
  // every warp scales h by the same power of two (from its own pass over the
  // interleaved words, conflict-free) and takes the 32 elements of vector
  // lane % LPR as f16 pairs
  float hs;
  {
    float hm = 0.f;
    for (int i = lane; i < I; i += 32) hm = fmaxf(hm, fabsf(s_h[i]));
    hm = segment_max<32>(hm);
    hs = pow2_scale_for(hm);
  }
  if (ok && !__all_sync(0xffffffffu, mbar_wait(bar_down, 0, p.status))) ok = false;
  if (ok) {
    uint32_t hr[16];
    const int hv = lane % LPR;
#pragma unroll
    for (int i = 0; i < 16; ++i) hr[i] = pack_f16x2(s_h[(2 * i) * LPR + hv] * hs, s_h[(2 * i + 1) * LPR + hv] * hs);
    const float ys = sd * gate / hs;
    for (int r = warp * RPS + lane / LPR; r < RPC; r += kTok1Warps * RPS) {
      const uint4 cv = lds128(dn_codes + r * DROW_C + 16 * (lane % LPR));
      const uint32_t s2 = *reinterpret_cast<const uint16_t*>(dn_scales + r * DROW_S + 2 * (lane % LPR));
      float acc = 0.f;
      dot32_strided<1, 16>(cv, s2, hr, &acc);
      acc = segment_sum<LPR>(acc);
      if (lane % LPR == 0) __stcg(part + r, acc * ys);
    }
  } else {
    for (int r = tid; r < RPC; r += blockDim.x) __stcg(part + r, 0.f);
  }

  // ---- P5: the last of the k + S CTAs of this row block sums the slots.
  // The barrier orders every thread's partial stores before thread 0's
  // arrival, whose release (cumulative) publishes them at GPU scope; its
  // acquire makes the other slots' partials visible to the last arriver, and
  // the barrier after it to all of its threads.
  __syncthreads();
  if (tid == 0) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(p.rb_count + rank) : "memory");
    const int last = old == static_cast<unsigned>(KS - 1);
    if (last) atomicExch(p.rb_count + rank, 0u);  // no other CTA of this launch touches it again
    s_last = last;
  }
  __syncthreads();
  if (s_last) {
    for (int r = tid; r < RPC; r += blockDim.x) {
      const int n = static_cast<int>(rank) * RPC + r;
      float y = 0.f;
      for (int j = 0; j < KS; ++j) y += __ldcg(p.partial + static_cast<size_t>(j) * D + n);
      if (p.residual != nullptr) y += bf16_bits_to_f32(__ldcg(p.residual + n));
      const __nv_bfloat16 b = __float2bfloat16_rn(y);
      p.out[n] = *reinterpret_cast<const uint16_t*>(&b);
    }
  }
  if (!p.trigger_early) pdl_trigger();
  // copies still in flight after a failed wait land before the CTA exits
  if (!ok && tid == 0) {
    mbar_wait(bar_x, 0, p.status);
    if (!shared && r1 > r0) mbar_wait(bar_rows, 0, p.status);
  }
  if (!ok && issued) {
    for (int c = tid; c < NCP; c += blockDim.x) mbar_wait(&bar_chunk[c], 0, p.status);
    if (tid == 0) mbar_wait(bar_down, 0, p.status);
  }
}

// Host side (tok1.cu): whether the cluster kernel serves (d, inter, E) on the
// current device (its shared memory fits, a 16-CTA cluster can be resident);
// with `launch`, also launches it for `t` on `st` and stores the launch status
// in *err.
bool tok1_dispatch(int d, int I, int E, bool launch, const Tok1Params* t, bool pdl, cudaStream_t st,
                   cudaError_t* err);

}  // namespace flint
