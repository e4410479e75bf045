// tokn.cuh -- the layer at decode batch 2..8 as persistent 16-CTA clusters.
//
// The grid is NC clusters of kTok1Cluster CTAs (as many as can be resident,
// at most the number of (expert) items a call can have). Every cluster routes
// the batch itself -- router logits on the register-fragment tensor cores,
// shared through distributed shared memory as in the one-token kernel, top-k
// per token, the grouping by expert (the experts the tokens selected,
// ascending, then the shared expert) -- and then takes the items a = cluster,
// cluster + NC, ... An item is one expert with its tokens (1..T of them): CTA
// r of the cluster owns units [r*I/16, (r+1)*I/16) of its gate/up and rows
// [r*d/16, (r+1)*d/16) of its down projection. Both go through the
// register-fragment tensor cores (mma.sync m16n8k16: 16 weight rows x the
// item's tokens as the 8 columns, the in-register NVFP4 decode of
// fused_tc.cuh), fed by per-warp rings of 256-column stages (one
// 128-byte-swizzled TMA box of codes, one box of scales) that run ahead across
// items. The cluster's items are cut into batches of consecutive items whose
// (token, slot) pairs fit the 8 rows of h; per batch:
//   gate/up  for each item: warp w < TL*KP takes tile w / KP (8 units = 16
//            rows) and K part w % KP (512 columns, two stages); the KP parts
//            of a tile meet in shared memory (named barrier per tile group,
//            double-buffered by item parity) and the group's first warp
//            applies SwiGLU and stores the item's h rows into every CTA of the
//            cluster (DSMEM; h double-buffered by batch parity)
//   cluster barrier: the batch's h is complete everywhere
//   h -> f16 with a power-of-two scale per row, in the B-fragment order
//   down     for each item: warp w < DT*DKP takes row tile w / DKP and K part
//            w % DKP (one 256-column stage); parts summed as above; the first
//            warp writes gate * s_d * W_d h for the item's (token, slot)
//            pairs: fp32 partials [token * (k+S) + slot][d] in the workspace
// so a batch costs one cluster barrier, not each item (with one per item the
// chain of barriers, not the weights' bytes, set the time).
//   arrival  after its last batch, one release/acquire atomic per CTA at its
//            row block's counter; the CTA that brings it to the number of
//            clusters adds, per token, the k + S partials of its rows in slot
//            order (+ residual), rounds to bf16 and resets the counter.
// No CTA waits on another cluster. Cluster barriers are reached by every CTA
// of a cluster on every path; every mbarrier wait is bounded; a warp whose
// wait gives up keeps taking every barrier (its work skipped).
#pragma once

#include <cuda.h>

#include "fused_tc.cuh"
#include "tok1.cuh"

namespace flint {

constexpr int kTnWarps = 16;
constexpr int kTnMaxTokens = 8;
constexpr int kTnMaxSlots = 3;         // ring slots per warp: 3 where they fit, else 2
constexpr int kTnStageCodes = 2048;    // 16 rows x 128 code bytes (256 columns), 128-byte swizzle
constexpr int kTnStageScales = 256;    // 16 rows x 16 scale bytes
constexpr int kTnMaxExperts = 256;     // router rows of a CTA fit the rings' 64 KiB

struct TokNParams {
  const uint16_t* x;         // [T][d] bf16
  const uint16_t* wr;        // [E][d] bf16
  const uint8_t* codes;      // packed E2M1 codes (L2 prefetch of upcoming items)
  const uint8_t* scales;     // packed E4M3 block scales
  long long cpe, spe;        // code / scale bytes per expert
  const float* tscale;       // [E+S][3]
  const uint16_t* residual;  // [T][d] bf16 or null
  uint16_t* out;             // [T][d] bf16
  int* status;
  unsigned* rb_count;        // [kTok1Cluster] arrival counters (workspace control block)
  float* partial;            // [T*(k+S)][d] gated partial outputs (workspace)
  int* ids;                  // [T][k] routed ids (workspace)
  float* gates;              // [T][k]
  int* ids_out;
  float* gates_out;
  int T, E, k, S;
  int input_norm;
};

// Gate/up: codes [E+S][2I][d/2] bytes, box 128 x 16 x 1, 128-byte swizzle;
// scales [E+S][2I][d/16], box 16 x 16 x 1. Down (from the expert's I*d/2-th
// code byte): codes [E+S][d][I/2], scales [E+S][d][I/16], same boxes.
struct TokNMaps {
  CUtensorMap gu_codes, gu_scales, dn_codes, dn_scales;
};

template <int D, int I>
struct TnShape {
  static constexpr int UPC = I / kTok1Cluster;   // gate/up units per CTA
  static constexpr int TL = UPC / 8;             // gate/up tiles (16 rows) per CTA
  static constexpr int KP = D / 512;             // gate/up K parts (512 columns)
  static constexpr int GU = TL * KP;             // gate/up warps
  static constexpr int RPC = D / kTok1Cluster;   // down rows per CTA
  static constexpr int DT = RPC / 16;            // down tiles per CTA
  static constexpr int DKP = I / 256;            // down K parts (256 columns)
  static constexpr int DN = DT * DKP;            // down warps
  static constexpr int XSTR = tc_b_stride(D), HSTR = tc_b_stride(I);
  static constexpr bool ok = (I >= 256) && (UPC % 8 == 0) && GU >= 1 && GU <= kTnWarps && DN >= 1 &&
                             DN <= kTnWarps && (TL + DT) <= 14;
};

// Row stride (bytes) of the router rows and of the tokens' bf16 x in shared
// memory: padded by 16 bytes, so that the eight rows one MMA fragment load
// touches fall in distinct banks (at the unpadded 2*d stride all 16 warps'
// fragment loads were 8-way bank conflicts).
__host__ __device__ constexpr int tn_row_stride(int D) { return 2 * D + 16; }
// Dynamic shared memory (after 1 KiB alignment slack): rings' codes and
// scales (the router rows use the codes area before the first item), x as
// f16 in the B-fragment order, h fp32 [2][8][I] (x's bf16 copy before the
// first item), h as f16 [8][HSTR] (the grouping's scratch before), the K-part
// partial sums of gate/up and down (2 buffers each), logits [8][E].
__host__ __device__ constexpr size_t tn_h32_bytes(int D, int I) {
  return (2 * kTnMaxTokens * static_cast<size_t>(I) * 4 > kTnMaxTokens * static_cast<size_t>(tn_row_stride(D)))
             ? 2 * kTnMaxTokens * static_cast<size_t>(I) * 4
             : kTnMaxTokens * static_cast<size_t>(tn_row_stride(D));
}
__host__ __device__ constexpr size_t tn_smem_bytes(int D, int I, int slots) {
  return 1024 + static_cast<size_t>(kTnWarps) * slots * (kTnStageCodes + kTnStageScales) +
         static_cast<size_t>(kTnMaxTokens) * tc_b_stride(D) + tn_h32_bytes(D, I) +
         ((static_cast<size_t>(kTnMaxTokens) * tc_b_stride(I) > 20 * kTnMaxExperts)
              ? static_cast<size_t>(kTnMaxTokens) * tc_b_stride(I)
              : 20 * kTnMaxExperts) +
         2 * 2 * static_cast<size_t>(kTnWarps) * 128 * 4 + static_cast<size_t>(kTnMaxTokens) * kTnMaxExperts * 4;
}
// Three slots hold a whole item's stages of a warp (two gate/up, one down), so
// the next item's stages are requested while this one is computed; with two,
// the second gate/up stage of each item was requested only at the end of the
// previous item and its whole load latency showed. The cap leaves room for
// the kernel's static shared memory within the 227 KiB an SM grants a CTA.
__host__ __device__ constexpr int tn_slots(int D, int I) {
  return tn_smem_bytes(D, I, 3) <= 227 * 1024 - 4096 ? 3 : 2;
}
__host__ __device__ constexpr size_t tn_smem_bytes(int D, int I) { return tn_smem_bytes(D, I, tn_slots(D, I)); }

// mma.sync m16n8k16, A row-major bf16, B column-major bf16, f32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t lds32(const void* p) { return *reinterpret_cast<const uint32_t*>(p); }


template <int D, int I>
__global__ void __launch_bounds__(kTnWarps * 32, 1) k_tokn(TokNParams p, const __grid_constant__ TokNMaps maps) {
  using SH = TnShape<D, I>;
  constexpr int CS = kTok1Cluster, TL = SH::TL, KP = SH::KP, GU = SH::GU, DKP = SH::DKP, DN = SH::DN;
  constexpr int RPC = SH::RPC, XSTR = SH::XSTR, HSTR = SH::HSTR;
  constexpr int NS = tn_slots(D, I);     // ring slots per warp
  constexpr int RS = tn_row_stride(D);   // padded bf16 row stride (router rows, x)
  constexpr int MAXB = kTnMaxTokens * kMaxTopK + 2;  // batch boundaries (items <= T*k + S)
  static_assert(kTok1Cluster * RS <= kTnWarps * NS * kTnStageCodes, "router rows fit the rings");
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[kTnWarps * kTnMaxSlots];
  __shared__ __align__(8) uint64_t bar_x, bar_rows;
  __shared__ int s_ids[kTnMaxTokens * kMaxTopK];
  __shared__ float s_gates[kTnMaxTokens * kMaxTopK];
  __shared__ int s_act[kTnMaxExperts + 1], s_off[kTnMaxExperts + 2], s_pair[kTnMaxTokens * (kMaxTopK + 1)];
  __shared__ int s_bstart[MAXB];
  __shared__ int s_nr, s_na, s_nb, s_fail, s_last;
  __shared__ float s_sig[kTnMaxTokens], s_irms[kTnMaxTokens], s_hsig[kTnMaxTokens];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = p.T, E = p.E, k = p.k, KS = k + p.S;
  const unsigned rank = cluster_rank();
  const int cl = static_cast<int>(cluster_index()), NC = static_cast<int>(gridDim.x) / CS;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* rcodes = base;                                             // [warp][slot][2048]
  uint8_t* rscales = rcodes + kTnWarps * NS * kTnStageCodes;          // [warp][slot][256]
  uint8_t* x16 = rscales + kTnWarps * NS * kTnStageScales;            // [8][XSTR]
  float* h32 = reinterpret_cast<float*>(x16 + kTnMaxTokens * XSTR);   // [2][8][I]
  uint8_t* h16 = reinterpret_cast<uint8_t*>(h32) + tn_h32_bytes(D, I);  // [8][HSTR]
  float* pgu = reinterpret_cast<float*>(h16 + ((kTnMaxTokens * HSTR > 20 * kTnMaxExperts) ? kTnMaxTokens * HSTR
                                                                                          : 20 * kTnMaxExperts));
  float* pdn = pgu + 2 * kTnWarps * 128;                               // [2][DN][128]
  float* s_logits = pdn + 2 * kTnWarps * 128;                          // [8][E]
  uint8_t* s_x = reinterpret_cast<uint8_t*>(h32);  // bf16 x, rows RS bytes apart, before the first item
  const int r0 = static_cast<int>(rank) * E / CS, r1 = (static_cast<int>(rank) + 1) * E / CS;
  uint64_t* wb = bars + warp * NS;

  // ---- P0: barriers; this CTA's router rows (one copy per row, padded rows)
  if (tid == 0) {
    for (int i = 0; i < kTnWarps * NS; ++i) mbar_init(&bars[i], 1);
    mbar_init(&bar_x, 1);
    mbar_init(&bar_rows, 1);
    fence_barrier_init();
    s_fail = 0;
  }
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar_rows, static_cast<uint32_t>(r1 - r0) * D * 2);
      mbar_arrive_expect_tx(&bar_x, static_cast<uint32_t>(T) * D * 2);
    }
    __syncwarp();
    if (lane < r1 - r0) bulk_g2s(rcodes + lane * RS, p.wr + static_cast<size_t>(r0 + lane) * D, D * 2, &bar_rows);
  }
  // release: a CTA's barrier and flag initialisation is visible to the remote
  // stores that follow the matching wait
  asm volatile("barrier.cluster.arrive.aligned;" ::: "memory");
  pdl_trigger();
  pdl_wait();
  if (warp == 0 && lane < T)
    bulk_g2s(s_x + lane * RS, p.x + static_cast<size_t>(lane) * D, D * 2, &bar_x);

  // ---- P1: per-token statistics (warp t), router logits of this CTA's rows
  // for every token into every CTA of the cluster; x as f16 in the
  // B-fragment order
  bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_x, 0, p.status));
  if (!__all_sync(0xffffffffu, mbar_wait(&bar_rows, 0, p.status))) ok = false;
  if (warp < T) {
    float amax = 0.f, ss = 0.f;
    for (int i = lane; i < D / 8; i += 32) {
      const uint4 v = lds128(s_x + warp * RS + 16 * i);
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
    if (lane == 0) {
      s_sig[warp] = pow2_scale_for(amax);
      s_irms[warp] = p.input_norm ? 1.f / sqrtf(ss / static_cast<float>(D) + kRmsEps) : 1.f;
    }
  }
  __syncthreads();
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");  // every CTA runs: remote stores allowed
  // a failed wait is made known to the whole cluster, so that every CTA of it
  // takes the same items (and cluster barriers) below
  if (!ok && lane < CS) st_cluster_u32(reinterpret_cast<unsigned*>(&s_fail), static_cast<unsigned>(lane), 1u);
  // router logits on the tensor cores: the CTA's rows r0..r1 (at most 16, the
  // MMA's M) x the batch's tokens (the 8 columns, unused ones repeat token 0),
  // K split over the 16 warps; bf16 products are exact, fp32 accumulation; the
  // warps' partial sums are added in warp order
  float* red = pgu;  // [16 warps][16 rows x 8 columns], free until the first item
  if (ok) {
    const int g = lane >> 2, t4 = lane & 3;
    const uint8_t* arow0 = rcodes + g * RS;
    const uint8_t* arow1 = rcodes + (g + 8) * RS;
    const uint8_t* brow = s_x + (g < T ? g : 0) * RS;
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    constexpr int KW = D / kTnWarps;
#pragma unroll
    for (int s = 0; s < KW / 16; ++s) {
      const int kb = (warp * KW + 16 * s + 2 * t4) * 2;  // byte offset of the lane's k pair
      mma_bf16_16816(c, lds32(arow0 + kb), lds32(arow1 + kb), lds32(arow0 + kb + 16), lds32(arow1 + kb + 16),
                     lds32(brow + kb), lds32(brow + kb + 16));
    }
    float* rw = red + warp * 128;
    rw[g * 8 + 2 * t4] = c[0];
    rw[g * 8 + 2 * t4 + 1] = c[1];
    rw[(g + 8) * 8 + 2 * t4] = c[2];
    rw[(g + 8) * 8 + 2 * t4 + 1] = c[3];
  }
  __syncthreads();
  if (ok && tid < 128) {
    const int rr = tid >> 3, t = tid & 7;
    if (rr < r1 - r0 && t < T) {
      float v = 0.f;
      for (int w = 0; w < kTnWarps; ++w) v += red[w * 128 + tid];
      const float logit = v * s_irms[t];
#pragma unroll 4
      for (int dst = 0; dst < CS; ++dst) st_cluster_f32(s_logits + t * E + r0 + rr, static_cast<unsigned>(dst), logit);
    }
  }
  for (int i = tid; i < kTnMaxTokens * (D / 8); i += blockDim.x) {
    const int t = i / (D / 8), c = i % (D / 8);
    uint4 o = make_uint4(0u, 0u, 0u, 0u);
    if (t < T) {
      const float sg = s_sig[t];
      const uint4 v = lds128(s_x + t * RS + 16 * c);
      o.x = bf16x2_to_f16x2_scaled(v.x, sg);
      o.y = bf16x2_to_f16x2_scaled(v.y, sg);
      o.z = bf16x2_to_f16x2_scaled(v.z, sg);
      o.w = bf16x2_to_f16x2_scaled(v.w, sg);
    }
    uint8_t* b = x16 + static_cast<size_t>(t) * XSTR + tc_b_offset(8 * c);
    *reinterpret_cast<uint32_t*>(b) = o.x;
    *reinterpret_cast<uint32_t*>(b + 16) = o.y;
    *reinterpret_cast<uint32_t*>(b + 32) = o.z;
    *reinterpret_cast<uint32_t*>(b + 48) = o.w;
  }

  // ---- P2: all logits everywhere; top-k per token (warp t), grouping, and
  // this cluster's items (a = cluster, cluster + NC, ...) cut into batches of
  // consecutive items whose (token, slot) pairs fit the 8 rows of h
  cluster_sync_all();
  if (s_fail) ok = false;
  if (warp < T && ok) {
    uint32_t code[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      code[i] = (e < E) ? max(route_code(s_logits[warp * E + e]), 1u) : 0u;
    }
    topk_rounds<8>(code, k, s_ids + warp * k, s_gates + warp * k, lane);
  }
  __syncthreads();
  if (ok) cta_grouping(s_ids, T, k, E, p.S, s_act, s_off, s_pair, &s_nr, &s_na, h16, p.status);
  __syncthreads();
  const int n_items = ok ? s_na : 0;
  const int n_my = n_items > cl ? (n_items - 1 - cl) / NC + 1 : 0;  // items cl, cl + NC, ...
  if (tid == 0) {
    int nb = 0, rows = 0;
    s_bstart[0] = 0;
    for (int it = 0; it < n_my; ++it) {
      const int a = cl + NC * it, ne = s_off[a + 1] - s_off[a];
      if (rows + ne > kTnMaxTokens && rows > 0) {
        s_bstart[++nb] = it;
        rows = 0;
      }
      rows += ne;
    }
    s_bstart[++nb] = n_my;
    s_nb = n_my > 0 ? nb : 0;
  }
  if (cl == 0 && rank == 0 && ok) {
    for (int i = tid; i < T * k; i += blockDim.x) {
      p.ids[i] = s_ids[i];
      p.gates[i] = s_gates[i];
      if (p.ids_out != nullptr) {
        p.ids_out[i] = s_ids[i];
        p.gates_out[i] = s_gates[i];
      }
    }
  }
  __syncthreads();
  const int n_batches = s_nb;
  // this warp's stage stream: per batch, the gate/up stages of its items (two
  // each when warp < GU), then their down stages (one each when warp < DN)
  const int gsw = warp < GU ? 2 : 0, dsw = warp < DN ? 1 : 0;
  const int n_st = n_my * (gsw + dsw);
  const int gt = warp / KP, gp = warp % KP;   // gate/up tile and K part
  const int dt = warp / DKP, dp = warp % DKP; // down tile and K part
  // issue cursor over the stream (batch, phase 0 gate/up / 1 down, item, stage)
  int cb = 0, cph = 0, cit = 0, ckk = 0;
  auto cur_norm = [&]() {  // move past phases without stages for this warp
    while (cb < n_batches) {
      if ((cph == 0 ? gsw : dsw) > 0 && cit < s_bstart[cb + 1]) return;
      if (cph == 0) {
        cph = 1;
      } else {
        cph = 0;
        ++cb;
      }
      cit = s_bstart[cb < n_batches ? cb : 0];
      ckk = 0;
    }
  };
  cur_norm();
  // a stage's three operations (the barrier's byte count, the codes box, the
  // scales box) go out from lanes 0, 1, 2 at once (the barrier's phase
  // completes only when the arrival and all bytes are in, whatever their order)
  auto issue = [&](int q) {  // lanes 0..2; the stage under the cursor
    const int e = s_act[cl + NC * cit], slot = q % NS;
    uint8_t* cs = rcodes + (warp * NS + slot) * kTnStageCodes;
    uint8_t* sc = rscales + (warp * NS + slot) * kTnStageScales;
    const bool gu = cph == 0;
    const int kc = gu ? gp * 512 + ckk * 256 : dp * 256;
    const int y = gu ? (static_cast<int>(rank) * TL + gt) * 16 : static_cast<int>(rank) * RPC + dt * 16;
    if (lane == 0) mbar_arrive_expect_tx(&wb[slot], kTnStageCodes + kTnStageScales);
    else if (lane == 1) tma_load_3d(cs, gu ? &maps.gu_codes : &maps.dn_codes, kc / 2, y, e, &wb[slot]);
    else tma_load_3d(sc, gu ? &maps.gu_scales : &maps.dn_scales, kc / 16, y, e, &wb[slot]);
  };
  auto issue_next = [&](int q) {  // whole warp: issue stage q, advance the cursor
    if (lane < 3) issue(q);
    if (++ckk == (cph == 0 ? gsw : dsw)) {
      ckk = 0;
      ++cit;
    }
    cur_norm();
  };
  int issued = 0;  // stages issued (the same in every lane)
  // the router rows in the codes area are read: order those reads first
  if (lane < 3) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  for (; issued < NS && issued < n_st; ++issued) issue_next(issued);
  int q = 0, q_fail = -1;  // stages consumed; first stage whose wait gave up
  auto wait_stage = [&]() -> bool {
    bool good = ok && (*reinterpret_cast<volatile int*>(&s_fail) == 0);
    good = __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
    if (good) good = __all_sync(0xffffffffu, mbar_wait(&wb[q % NS], (q / NS) & 1, p.status));
    if (!good) {
      if (ok) q_fail = q;
      ok = false;
      if (lane == 0) s_fail = 1;
    }
    return good;
  };
  auto release_stage = [&]() {  // the slot's data is read: refill it
    __syncwarp();
    if (ok && issued < n_st) {
      if (lane < 3) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue_next(issued);
      ++issued;
    }
    ++q;
  };
  const int g = lane >> 2, t4 = lane & 3;

  int gitem = 0;  // items before this batch (parity of the partial-sum buffers)
  for (int bt = 0; bt < n_batches; ++bt) {
    const int i0 = s_bstart[bt], i1 = s_bstart[bt + 1];
    float* hb = h32 + static_cast<size_t>(bt & 1) * kTnMaxTokens * I;  // h rows of this batch
    // ---- gate/up + SwiGLU of the batch's items; item it's tokens are h rows
    // row0 .. row0 + ne - 1, stored into every CTA of the cluster
    int row0 = 0;
    for (int it = i0; it < i1; ++it) {
      const int a = cl + NC * it, buf = (gitem + it - i0) & 1;
      const int e = s_act[a], pb = s_off[a], ne = s_off[a + 1] - pb;
      if (warp < GU) {
        const float sgt = __ldg(p.tscale + 3 * e + 0), sut = __ldg(p.tscale + 3 * e + 1);
        // the lane's ldmatrix row: the token of column lane % 8 (unused columns repeat column 0)
        const int my_pair = s_pair[pb + ((lane & 7) < ne ? (lane & 7) : 0)];
        const uint8_t* xrow = x16 + static_cast<size_t>(my_pair >> 8) * XSTR;
        const int rg = 2 * tc_unit_of(g), ru = rg + 1;
        float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
        for (int s = 0; s < 2; ++s) {
          if (wait_stage()) {
            const uint8_t* cs = rcodes + (warp * NS + (q % NS)) * kTnStageCodes;
            const uint8_t* ss = rscales + (warp * NS + (q % NS)) * kTnStageScales;
#pragma unroll
            for (int seg = 0; seg < 2; ++seg) {
              uint32_t b[16];
              tc_load_b(xrow, (gp * 4 + s * 2 + seg) * 256, lane, b);
              const uint4 ca = lds128(tc_code_chunk(cs, rg, seg, t4)), cb2 = lds128(tc_code_chunk(cs, ru, seg, t4));
              const uint32_t sa = *reinterpret_cast<const uint16_t*>(ss + rg * 16 + seg * 8 + 2 * t4);
              const uint32_t sb = *reinterpret_cast<const uint16_t*>(ss + ru * 16 + seg * 8 + 2 * t4);
              tc_segment(acc, acc1, ca, cb2, sa, sb, b);
            }
          }
          release_stage();
        }
        float* pp = pgu + (static_cast<size_t>(buf) * kTnWarps + gt * KP) * 128;
#pragma unroll
        for (int r = 0; r < 4; ++r) pp[gp * 128 + r * 32 + lane] = acc[r] + acc1[r];
        if constexpr (KP > 1) named_sync(1 + gt, 32 * KP);
        else __syncwarp();
        if (gp == 0) {
          float v[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            v[r] = 0.f;
#pragma unroll
            for (int k2 = 0; k2 < KP; ++k2) v[r] += pp[k2 * 128 + r * 32 + lane];
          }
          const int u = (static_cast<int>(rank) * TL + gt) * 8 + tc_unit_of(g);  // unit within the expert
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int col = 2 * t4 + h2;
            if (col < ne) {
              const int tok = s_pair[pb + col] >> 8;
              const float f = s_irms[tok] / s_sig[tok];
              const float hv = swiglu(v[h2] * f * sgt, v[2 + h2] * f * sut);
#pragma unroll 4
              for (int dst = 0; dst < CS; ++dst)
                st_cluster_f32(hb + (row0 + col) * I + u, static_cast<unsigned>(dst), hv);
            }
          }
        }
      }
      row0 += ne;
    }
    // ---- the batch's h rows are complete in every CTA of the cluster (the
    // other buffer is written only after the next batch's barrier, which every
    // CTA reaches after its conversion below)
    cluster_sync_all();
    // h -> f16 in the B-fragment order with a power-of-two scale per row
    // (warp n: row n)
    if (warp < row0) {
      const float* hr = hb + static_cast<size_t>(warp) * I;
      float hm = 0.f;
      for (int i = lane; i < I; i += 32) hm = fmaxf(hm, fabsf(hr[i]));
      hm = segment_max<32>(hm);
      const float hs = pow2_scale_for(hm);
      if (lane == 0) s_hsig[warp] = hs;
      for (int i = lane; i < I / 2; i += 32) {
        const uint32_t v = pack_f16x2(hr[2 * i] * hs, hr[2 * i + 1] * hs);
        *reinterpret_cast<uint32_t*>(h16 + static_cast<size_t>(warp) * HSTR + tc_b_offset(2 * i)) = v;
      }
    }
    __syncthreads();
    // ---- down of the batch's items against their h rows
    row0 = 0;
    for (int it = i0; it < i1; ++it) {
      const int a = cl + NC * it, buf = (gitem + it - i0) & 1;
      const int e = s_act[a], pb = s_off[a], ne = s_off[a + 1] - pb;
      if (warp < DN) {
        const float sdt = __ldg(p.tscale + 3 * e + 2);
        const uint8_t* hrow = h16 + static_cast<size_t>(row0 + ((lane & 7) < ne ? (lane & 7) : 0)) * HSTR;
        float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
        if (wait_stage()) {
          const uint8_t* cs = rcodes + (warp * NS + (q % NS)) * kTnStageCodes;
          const uint8_t* ss = rscales + (warp * NS + (q % NS)) * kTnStageScales;
#pragma unroll
          for (int seg = 0; seg < 2; ++seg) {
            uint32_t b[16];
            tc_load_b(hrow, (dp * 2 + seg) * 256, lane, b);
            const uint4 ca = lds128(tc_code_chunk(cs, g, seg, t4)), cb2 = lds128(tc_code_chunk(cs, g + 8, seg, t4));
            const uint32_t sa = *reinterpret_cast<const uint16_t*>(ss + g * 16 + seg * 8 + 2 * t4);
            const uint32_t sb = *reinterpret_cast<const uint16_t*>(ss + (g + 8) * 16 + seg * 8 + 2 * t4);
            tc_segment(acc, acc1, ca, cb2, sa, sb, b);
          }
        }
        release_stage();
        float* pp = pdn + (static_cast<size_t>(buf) * kTnWarps + dt * DKP) * 128;
#pragma unroll
        for (int r = 0; r < 4; ++r) pp[dp * 128 + r * 32 + lane] = acc[r] + acc1[r];
        if constexpr (DKP > 1) named_sync(1 + TL + dt, 32 * DKP);
        else __syncwarp();
        if (dp == 0) {
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            float v = 0.f;
#pragma unroll
            for (int k2 = 0; k2 < DKP; ++k2) v += pp[k2 * 128 + r * 32 + lane];
            const int col = 2 * t4 + (r & 1), row = static_cast<int>(rank) * RPC + dt * 16 + g + 8 * (r >> 1);
            if (col < ne && ok) {
              const int pr = s_pair[pb + col], tok = pr >> 8, j = pr & 0xFF;
              const float gate = j < k ? s_gates[tok * k + j] : 1.f;
              __stcg(p.partial + static_cast<size_t>(tok * KS + j) * D + row, v * sdt * gate / s_hsig[row0 + col]);
            }
          }
        }
      }
      row0 += ne;
    }
    gitem += i1 - i0;
  }
  // copies still in flight after a failed wait land before the CTA goes on
  if (!ok && lane == 0 && q_fail >= 0)
    for (int k2 = q_fail; k2 < issued; ++k2) mbar_wait(&wb[k2 % NS], (k2 / NS) & 1, p.status);
  if (!ok && tid == 0) {
    mbar_wait(&bar_x, 0, p.status);
    mbar_wait(&bar_rows, 0, p.status);
  }
  // ---- arrival at this CTA's row block: once per CTA, whatever happened
  // above, so the counter returns to zero; the CTA that brings it to the
  // number of clusters adds the row block's partials
  __syncthreads();
  if (tid == 0) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(p.rb_count + rank) : "memory");
    const int last = old == static_cast<unsigned>(NC - 1);
    if (last) atomicExch(p.rb_count + rank, 0u);
    s_last = last;
  }
  __syncthreads();
  if (s_last) {
    for (int idx = tid; idx < T * RPC; idx += blockDim.x) {
      const int t = idx / RPC, n = static_cast<int>(rank) * RPC + idx % RPC;
      float y = 0.f;
      for (int j = 0; j < KS; ++j) y += __ldcg(p.partial + static_cast<size_t>(t * KS + j) * D + n);
      const size_t o = static_cast<size_t>(t) * D + n;
      if (p.residual != nullptr) y += bf16_bits_to_f32(__ldcg(p.residual + o));
      const __nv_bfloat16 bv = __float2bfloat16_rn(y);
      p.out[o] = *reinterpret_cast<const uint16_t*>(&bv);
    }
  }
}

// Host side (tokn.cu): whether the kernel serves (d, inter, E, T) on the
// current device and, with `launch`, its launch for `t` on `st` (status in
// *err). `maps` as TokNMaps.
bool tokn_dispatch(int d, int I, int E, int T, bool launch, const TokNParams* t, const TokNMaps* maps, bool pdl,
                   cudaStream_t st, cudaError_t* err);

}  // namespace flint
