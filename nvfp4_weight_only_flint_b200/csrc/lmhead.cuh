// lmhead.cuh -- the 4-bit output head: a dense NVFP4 matrix [V][d] times the
// tokens' bf16 hidden states, fp32 logits out (W4A16, as the experts).
//
// One persistent CTA per SM streams a contiguous range of rows through a ring
// of bulk-copy stages (16 rows of codes + their block scales per stage); warp
// w takes row w of every stage. Every token's x is staged once per CTA as f16
// after a per-token power-of-two scale and held in registers (one or two
// tokens: a decode GEMV) while the stages' rows stream past (the decode of
// cvt.rn.f16x2.e2m1x2 and the block scale in f32, fma.rn.f32.f16 products
// exact, fp32 accumulation). The tensor scale and 1/sigma are applied once per
// logit. The op is a pure stream: its roofline is HBM.
#pragma once

#include "common.cuh"

namespace flint {

constexpr int kLmWarps = 16;
constexpr int kLmRows = 16;     // rows per stage (one per warp)
constexpr int kLmMaxTokens = 2;   // tokens per call (one at d = 4096)
constexpr int kLmMaxStages = 8;

struct LmHeadParams {
  const uint16_t* x;      // [T][d] bf16
  const uint8_t* codes;   // [V][d/2]
  const uint8_t* scales;  // [V][d/16]
  const float* tscale;    // [1]
  float* out;             // [T][V]
  int* status;            // status word (bounded waits)
  int T, V;
  int stages;             // ring depth
};

__host__ __device__ constexpr size_t lm_stage_bytes(int D) { return static_cast<size_t>(kLmRows) * (D / 2 + D / 16); }
__host__ __device__ constexpr size_t lm_smem_bytes(int D, int stages) {
  return static_cast<size_t>(stages) * lm_stage_bytes(D) + static_cast<size_t>(kLmMaxTokens) * D * 2;
}

// Host side (lmhead.cu): launches the head for `p` on `st` (d one of 512,
// 1024, 2048, 4096) and returns the launch status.
cudaError_t lm_head_launch(int d, const LmHeadParams& p, cudaStream_t st);

}  // namespace flint
