// lmhead.cu -- the 4-bit output head kernel and its launch (see lmhead.cuh).

#include "lmhead.cuh"

namespace flint {
namespace {

template <int D, int T>
__global__ void __launch_bounds__(kLmWarps * 32, 1) k_lm_head(LmHeadParams p) {
  constexpr int VPR = D / 32;                  // 16-byte code vectors per row
  constexpr int XV = VPR >= 32 ? VPR / 32 : 1;  // vectors per lane
  constexpr int ROWC = D / 2, ROWS = D / 16;
  constexpr int STC = kLmRows * ROWC;          // code bytes of a stage
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full[kLmMaxStages], empty[kLmMaxStages];
  __shared__ float s_f[kLmMaxTokens];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int NS = p.stages, G = gridDim.x, c = blockIdx.x;
  const size_t stb = lm_stage_bytes(D);
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + NS * stb);
  const int row0 = static_cast<int>(static_cast<long long>(c) * p.V / G);
  const int row1 = static_cast<int>(static_cast<long long>(c + 1) * p.V / G);
  const int n_st = (row1 - row0 + kLmRows - 1) / kLmRows;

  auto issue = [&](int i) {  // stage i of this CTA's rows into slot i % NS
    const int r = row0 + i * kLmRows, n = min(kLmRows, row1 - r);
    uint8_t* st = smem + (i % NS) * stb;
    mbar_arrive_expect_tx(&full[i % NS], n * (ROWC + ROWS));
    bulk_g2s(st, p.codes + static_cast<long long>(r) * ROWC, n * ROWC, &full[i % NS]);
    bulk_g2s(st + STC, p.scales + static_cast<long long>(r) * ROWS, n * ROWS, &full[i % NS]);
  };
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kLmWarps);
    }
    fence_barrier_init();
    for (int i = 0; i < NS && i < n_st; ++i) issue(i);  // weights do not depend on earlier kernels
  }
  pdl_wait();
  // the tokens' x, scaled per token by a power of two into f16 (warp t: token t)
  if (warp < T) {
    const uint4* src = reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(warp) * D);
    float amax = 0.f;
    for (int i = lane; i < D / 8; i += 32) {
      const uint4 v = __ldcg(src + i);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
        amax = fmaxf(amax, fmaxf(fabsf(bf16_bits_to_f32(w4[q] & 0xFFFFu)), fabsf(__uint_as_float(w4[q] & 0xFFFF0000u))));
    }
    amax = segment_max<32>(amax);
    const float sg = pow2_scale_for(amax);
    if (lane == 0) s_f[warp] = __ldg(p.tscale) / sg;
    for (int i = lane; i < D / 8; i += 32) {
      const uint4 v = __ldcg(src + i);
      uint4 o;
      o.x = pack_f16x2(bf16_bits_to_f32(v.x & 0xFFFFu) * sg, __uint_as_float(v.x & 0xFFFF0000u) * sg);
      o.y = pack_f16x2(bf16_bits_to_f32(v.y & 0xFFFFu) * sg, __uint_as_float(v.y & 0xFFFF0000u) * sg);
      o.z = pack_f16x2(bf16_bits_to_f32(v.z & 0xFFFFu) * sg, __uint_as_float(v.z & 0xFFFF0000u) * sg);
      o.w = pack_f16x2(bf16_bits_to_f32(v.w & 0xFFFFu) * sg, __uint_as_float(v.w & 0xFFFF0000u) * sg);
      *reinterpret_cast<uint4*>(xs + static_cast<size_t>(warp) * D + 8 * i) = o;
    }
  }
  __syncthreads();
  pdl_trigger();
  // x of the lane's vectors v = lane + 32 j (lanes beyond VPR repeat)
  const int xl = lane % VPR;
  uint32_t xr[T][XV][16];
#pragma unroll
  for (int t = 0; t < T; ++t)
#pragma unroll
    for (int j = 0; j < XV; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 v = lds128(xs + static_cast<size_t>(t) * D + (xl + 32 * j) * 32 + 8 * q);
        xr[t][j][4 * q + 0] = v.x;
        xr[t][j][4 * q + 1] = v.y;
        xr[t][j][4 * q + 2] = v.z;
        xr[t][j][4 * q + 3] = v.w;
      }
  float f[T];
#pragma unroll
  for (int t = 0; t < T; ++t) f[t] = s_f[t];

  bool ok = true;
  int i = 0;
  for (; i < n_st && ok; ++i) {
    const int slot = i % NS;
    if (!__all_sync(0xffffffffu, mbar_wait(&full[slot], (i / NS) & 1, p.status))) {
      ok = false;
      break;
    }
    const int r = row0 + i * kLmRows + warp;
    if (r < row1) {
      const uint8_t* st = smem + slot * stb;
      float acc[T];
#pragma unroll
      for (int t = 0; t < T; ++t) acc[t] = 0.f;
      if (lane < VPR) {
#pragma unroll
        for (int j = 0; j < XV; ++j) {
          const int v = xl + 32 * j;
          const uint4 cv = lds128(st + warp * ROWC + 16 * v);
          const uint32_t s2 = *reinterpret_cast<const uint16_t*>(st + STC + warp * ROWS + 2 * v);
#pragma unroll
          for (int t = 0; t < T; ++t) dot32_strided<1, 16>(cv, s2, xr[t][j], &acc[t]);
        }
      }
#pragma unroll
      for (int t = 0; t < T; ++t) {
        const float s = warp_sum(acc[t]);
        if (lane == 0) p.out[static_cast<size_t>(t) * p.V + r] = s * f[t];
      }
    }
    __syncwarp();
    if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(&empty[slot])) : "memory");
    // the producer refills the slot once every warp is done with it
    if (tid == 0 && i + NS < n_st) {
      if (!mbar_wait(&empty[slot], (i / NS) & 1, p.status)) {
        ok = false;
      } else {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue(i + NS);
      }
    }
  }
  // copies still in flight after a failed wait land before the CTA exits
  if (!ok && tid == 0) {
    const int issued = min(n_st, i + NS);
    for (int k = i; k < issued; ++k) mbar_wait(&full[k % NS], (k / NS) & 1, p.status);
  }
}

template <int D, int T>
cudaError_t launch_dt(const LmHeadParams& p, cudaStream_t st) {
  auto kern = k_lm_head<D, T>;
  const size_t smem = lm_smem_bytes(D, p.stages);
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
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int D>
cudaError_t launch_d(const LmHeadParams& p, cudaStream_t st) {
  return p.T == 1 ? launch_dt<D, 1>(p, st) : launch_dt<D, 2>(p, st);
}

}  // namespace

cudaError_t lm_head_launch(int d, const LmHeadParams& p, cudaStream_t st) {
  switch (d) {
    case 512: return launch_d<512>(p, st);
    case 1024: return launch_d<1024>(p, st);
    case 2048: return launch_d<2048>(p, st);
    default: return launch_dt<4096, 1>(p, st);
  }
}

}  // namespace flint
