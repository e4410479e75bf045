// lmhead.cu -- the 4-bit output head kernel and its launch (see lmhead.cuh).

#include "lmhead.cuh"

namespace flint {
namespace {

template <int D>
__global__ void __launch_bounds__(kLmWarps * 32, 1) k_lm_head(LmHeadParams p, const __grid_constant__ LmMaps maps) {
  constexpr int KP = D / 512;          // K parts (warps) per tile
  constexpr int TPI = kLmWarps / KP;   // tiles in flight per CTA
  constexpr int XSTR = tc_b_stride(D);
  constexpr int NS = lm_stages(D);
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[kLmWarps * NS];
  __shared__ int s_fail;
  __shared__ float s_f[kLmMaxTokens];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* codes = base;                                              // [warp][stage][4096], 1 KiB aligned
  uint8_t* scales = codes + kLmWarps * NS * kTcStageCodes;             // [warp][stage][512]
  uint8_t* x16 = scales + kLmWarps * NS * kTcStageScales;              // [8][XSTR] f16, B-fragment order
  float* part = reinterpret_cast<float*>(x16 + kLmMaxTokens * XSTR);   // [TPI groups][2][KP][128]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n_tiles = (p.V + 15) / 16, G = gridDim.x, c = blockIdx.x;
  const int tile0 = static_cast<int>(static_cast<long long>(c) * n_tiles / G);
  const int L = static_cast<int>(static_cast<long long>(c + 1) * n_tiles / G) - tile0;
  const int kp = warp % KP, m = warp / KP;
  const int n_q = L > m ? (L - 1 - m) / TPI + 1 : 0;  // this warp's stages: local tile m + TPI*q, part kp
  uint64_t* wb = bars + warp * NS;

  auto issue = [&](int q) {
    const int slot = q % NS, y = (tile0 + m + TPI * q) * 16;
    uint8_t* cs = codes + (warp * NS + slot) * kTcStageCodes;
    mbar_arrive_expect_tx(&wb[slot], kTcStageCodes + kTcStageScales);
    tma_load_2d(cs, &maps.codes, kp * 256, y, &wb[slot]);
    tma_load_2d(cs + 2048, &maps.codes, kp * 256 + 128, y, &wb[slot]);
    tma_load_2d(scales + (warp * NS + slot) * kTcStageScales, &maps.scales, kp * 32, y, &wb[slot]);
  };
  if (tid == 0) {
    for (int i = 0; i < kLmWarps * NS; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
  }
  if (tid == 0) s_fail = 0;
  __syncthreads();
  int issued = 0;
  if (lane == 0)  // weights do not depend on earlier kernels
    for (; issued < NS && issued < n_q; ++issued) issue(issued);
  issued = __shfl_sync(0xffffffffu, issued, 0);
  pdl_wait();
  // the tokens' x as f16 after a power-of-two scale each (warp t: token t);
  // rows of unused columns are zero
  if (warp < kLmMaxTokens) {
    const int t = warp;
    const uint4* src = reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(t) * D);
    float amax = 0.f;
    if (t < p.T) {
      for (int i = lane; i < D / 8; i += 32) {
        const uint4 v = __ldcg(src + i);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
          amax = fmaxf(amax, fmaxf(fabsf(bf16_bits_to_f32(w4[q] & 0xFFFFu)), fabsf(__uint_as_float(w4[q] & 0xFFFF0000u))));
      }
    }
    amax = segment_max<32>(amax);
    const float sg = pow2_scale_for(amax);
    if (lane == 0) s_f[t] = (t < p.T) ? __ldg(p.tscale) / sg : 0.f;
    for (int i = lane; i < D / 8; i += 32) {
      uint4 o = make_uint4(0u, 0u, 0u, 0u);
      if (t < p.T) {
        const uint4 v = __ldcg(src + i);
        o.x = pack_f16x2(bf16_bits_to_f32(v.x & 0xFFFFu) * sg, __uint_as_float(v.x & 0xFFFF0000u) * sg);
        o.y = pack_f16x2(bf16_bits_to_f32(v.y & 0xFFFFu) * sg, __uint_as_float(v.y & 0xFFFF0000u) * sg);
        o.z = pack_f16x2(bf16_bits_to_f32(v.z & 0xFFFFu) * sg, __uint_as_float(v.z & 0xFFFF0000u) * sg);
        o.w = pack_f16x2(bf16_bits_to_f32(v.w & 0xFFFFu) * sg, __uint_as_float(v.w & 0xFFFF0000u) * sg);
      }
      // elements 8i + 2j, +1 (j = 0..3) sit 16 bytes apart in the B-fragment order
      uint8_t* b = x16 + static_cast<size_t>(t) * XSTR + tc_b_offset(8 * i);
      *reinterpret_cast<uint32_t*>(b) = o.x;
      *reinterpret_cast<uint32_t*>(b + 16) = o.y;
      *reinterpret_cast<uint32_t*>(b + 32) = o.z;
      *reinterpret_cast<uint32_t*>(b + 48) = o.w;
    }
  }
  __syncthreads();
  pdl_trigger();
  float f[2];
  const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
  for (int h = 0; h < 2; ++h) f[h] = s_f[2 * t4 + h];
  const uint8_t* xrow = x16 + static_cast<size_t>(lane & 7) * XSTR;

  // The KP warps of a tile group take the same steps in lockstep (a named
  // barrier per step, so no warp runs ahead of its group); step q's partial
  // sums use buffer q & 1 of the group, which the group's part-0 warp adds in
  // part order after the barrier; the next step's barrier orders that read
  // before the buffer is written again two steps later. A warp whose wait
  // gives up keeps taking every step and barrier (later waits are skipped)
  // so that its group never waits on it.
  bool ok = true;
  int q_fail = n_q;  // stages [q_fail, issued) may still be in flight after a failure
  float* gp = part + static_cast<size_t>(m) * 2 * KP * 128;  // [2][KP][128]
  for (int q = 0; q < n_q; ++q) {
    const int slot = q % NS;
    const int fail_now = __shfl_sync(0xffffffffu, *reinterpret_cast<volatile int*>(&s_fail), 0);
    if (ok && fail_now == 0) {
      if (!__all_sync(0xffffffffu, mbar_wait(&wb[slot], (q / NS) & 1, p.status))) {
        ok = false;
        q_fail = q;
        if (lane == 0) s_fail = 1;
      }
    } else if (ok) {
      ok = false;  // another warp's wait gave up: skip the rest
      q_fail = q;
    }
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
    if (ok) {
      const uint8_t* cs = codes + (warp * NS + slot) * kTcStageCodes;
      const uint8_t* ss = scales + (warp * NS + slot) * kTcStageScales;
#pragma unroll 2
      for (int seg = 0; seg < 4; ++seg) {
        uint32_t b[16];
        tc_load_b(xrow, (kp * 4 + seg) * 256, lane, b);
        const uint4 ca = lds128(tc_code_chunk(cs, g, seg, t4)), cb = lds128(tc_code_chunk(cs, g + 8, seg, t4));
        const uint32_t sa = *reinterpret_cast<const uint16_t*>(ss + g * 32 + seg * 8 + 2 * t4);
        const uint32_t sb = *reinterpret_cast<const uint16_t*>(ss + (g + 8) * 32 + seg * 8 + 2 * t4);
        tc_segment(acc, acc1, ca, cb, sa, sb, b);
      }
      __syncwarp();
      if (q + NS < n_q && lane == 0) {  // the slot is read: refill it
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue(q + NS);
        ++issued;
      }
    }
    float* pp = gp + (q & 1) * KP * 128;
#pragma unroll
    for (int r = 0; r < 4; ++r) pp[kp * 128 + r * 32 + lane] = acc[r] + acc1[r];
    if constexpr (KP > 1) asm volatile("bar.sync %0, %1;" ::"r"(m + 1), "r"(32 * KP) : "memory");
    else __syncwarp();
    if (kp == 0) {
      const int row_base = (tile0 + m + TPI * q) * 16;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        float v = 0.f;
#pragma unroll
        for (int k2 = 0; k2 < KP; ++k2) v += pp[k2 * 128 + r * 32 + lane];
        const int row = row_base + g + 8 * (r >> 1), col = 2 * t4 + (r & 1);
        if (ok && col < p.T && row < p.V) p.out[static_cast<size_t>(col) * p.V + row] = v * f[r & 1];
      }
    }
  }
  // copies still in flight after a failed wait land before the CTA exits
  if (!ok && lane == 0)
    for (int k2 = q_fail; k2 < issued; ++k2) mbar_wait(&wb[k2 % NS], (k2 / NS) & 1, p.status);
}

template <int D>
cudaError_t launch_d(const LmHeadParams& p, const LmMaps& maps, cudaStream_t st) {
  auto kern = k_lm_head<D>;
  const size_t smem = lm_smem_bytes(D);
  cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(kern), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sms);
  cfg.blockDim = dim3(kLmWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p, maps);
}

}  // namespace

cudaError_t lm_head_launch(int d, const LmHeadParams& p, const LmMaps& maps, cudaStream_t st) {
  switch (d) {
    case 512: return launch_d<512>(p, maps, st);
    case 1024: return launch_d<1024>(p, maps, st);
    case 2048: return launch_d<2048>(p, maps, st);
    default: return launch_d<4096>(p, maps, st);
  }
}

}  // namespace flint
