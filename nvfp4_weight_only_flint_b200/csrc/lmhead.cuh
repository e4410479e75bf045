// lmhead.cuh -- the 4-bit output head: a dense NVFP4 matrix [V][d] times the
// tokens' bf16 hidden states, fp32 logits out (W4A16, as the experts).
//
// A pure stream (its roofline is HBM), so the point is to move the 173 MB of
// the Flint head at full bandwidth with few instructions per weight: a
// CUDA-core loop spends about four instructions per weight (decode, unpack,
// multiply-add) and is issue-bound near half the bandwidth. Here the weights
// go through the register-fragment tensor-core path of the persistent layer
// kernel (fused_tc.cuh): one persistent CTA per SM takes a contiguous range
// of 16-row tiles; a tile's K range is cut into parts of 512 columns, one
// per warp (d/512 warps per tile), each part arriving in the warp's own ring
// as two 128-byte-swizzled TMA boxes of codes and one box of scales; the warp
// decodes them into mma.sync A fragments (exact e2m1 * e4m3 in f16) against
// the tokens' x (f16 after a power-of-two scale per token, up to 8 tokens as
// the 8 MMA columns, read with ldmatrix) and accumulates in fp32. The parts'
// partial sums meet in shared memory and the last warp to arrive adds them
// in part order (deterministic) and applies the tensor scale and 1/sigma.
#pragma once

#include <cuda.h>

#include "fused_tc.cuh"

namespace flint {

constexpr int kLmWarps = 16;
constexpr int kLmMaxTokens = 8;
// ring depth per warp (stages of 16 rows x 512 K): two, one at d = 4096 where
// the staged x takes twice the room
__host__ __device__ constexpr int lm_stages(int D) { return D == 4096 ? 1 : 2; }

struct LmHeadParams {
  const uint16_t* x;      // [T][d] bf16
  const float* tscale;    // [1]
  float* out;             // [T][V]
  int* status;            // status word (bounded waits)
  int T, V;
};

// Codes [V][d/2] bytes: box 128 x 16 with the 128-byte swizzle; scales
// [V][d/16] bytes: box 32 x 16.
struct LmMaps {
  CUtensorMap codes;
  CUtensorMap scales;
};

// Dynamic shared memory: 1 KiB alignment slack, the warps' rings, the staged
// x (8 rows), and the K-part partial sums (2 * 16 warps' fragments).
__host__ __device__ constexpr size_t lm_smem_bytes(int D) {
  return 1024 + static_cast<size_t>(kLmWarps) * lm_stages(D) * (kTcStageCodes + kTcStageScales) +
         static_cast<size_t>(kLmMaxTokens) * tc_b_stride(D) + static_cast<size_t>(2 * kLmWarps) * 128 * sizeof(float);
}

// Host side (lmhead.cu): launches the head for `p` on `st` (d one of 512,
// 1024, 2048, 4096) and returns the launch status.
cudaError_t lm_head_launch(int d, const LmHeadParams& p, const LmMaps& maps, cudaStream_t st);

}  // namespace flint
