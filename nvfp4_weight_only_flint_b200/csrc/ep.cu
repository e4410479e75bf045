// ep.cu -- expert-parallel dispatch and combine for one MoE layer sharded over
// the GPUs of one node ("[Model] Add Flint (RecursiveSI/flint)", section "What
// happened": the tuned path is tensor-parallel degree 1, expert parallelism is
// left on the stock layers; the layer is the "Recursive Flint: 125 tok/s on
// an M4 Pro" architecture table's 256 routed experts, 6 per token, 1 shared).
//
// Rank r of R holds routed experts [r E/R, (r+1) E/R) plus the shared expert,
// packed as E/R + 1 experts (shared last), so on every rank the shared expert
// is local id E/R. A token's (token, slot) pairs go to the rank that holds the
// slot's expert; its shared-expert pair goes to its own rank. Every rank then
// runs one routed call (flint_moe_forward_routed, top_k = 1) over all the rows
// it received, each row scaled by its gate, and sends the rows back; the home
// rank sums a token's rows.
//
// k_ep_plan: one CTA of 1024 threads. A stable counting sort of the T (k + S)
// pairs by destination rank (order within a rank = pair order t (k + S) + j):
// each thread takes a contiguous run of pairs, counts per rank, the per-rank
// counts are scanned over threads, and a second pass places the pairs.
// k_ep_gather: the send rows, 16-byte vectors over the whole grid.
// k_ep_combine: out[t] = bf16(sum_j y[pair_pos[t][j]] + residual[t]), fp32.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "flint_moe.h"
#include "common.cuh"

namespace flint {
namespace {

constexpr int kEpThreads = 1024;
constexpr int kEpMaxRanks = 8;
constexpr int kEpMaxSlots = 9;  // top_k <= 8 plus the shared expert

struct PlanParams {
  const int32_t* ids;    // [T][k]
  const float* gates;    // [T][k]
  int32_t* send_ids;     // [P] local expert id on the destination rank
  float* send_gates;     // [P]
  int32_t* send_token;   // [P] source token of each send row
  int32_t* send_counts;  // [R]
  int32_t* pair_pos;     // [T][k+S] send position of each pair (-1: dropped)
  int32_t* status;
  int T, k, S, E, R, rank;
};

__device__ __forceinline__ int pair_dest(const PlanParams& p, int i, int& lid, float& g, bool record) {
  const int slots = p.k + p.S;
  const int t = i / slots, j = i % slots;
  const int el = p.E / p.R;
  if (j >= p.k) {  // the shared expert: local id E/R on the token's own rank
    lid = el;
    g = 1.f;
    return p.rank;
  }
  const int e = p.ids[t * p.k + j];
  if (e < 0 || e >= p.E) {
    if (record && p.status != nullptr) atomicOr(p.status, FLINT_DEVCHECK_EXPERT_ID);
    return -1;
  }
  lid = e % el;
  g = p.gates[t * p.k + j];
  return e / el;
}

__global__ void __launch_bounds__(kEpThreads) k_ep_plan(PlanParams p) {
  __shared__ int s_cnt[kEpMaxRanks][kEpThreads];
  __shared__ int s_base[kEpMaxRanks];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int P = p.T * (p.k + p.S);
  const int per = (P + kEpThreads - 1) / kEpThreads;
  const int i0 = min(P, tid * per), i1 = min(P, i0 + per);
  int c[kEpMaxRanks];
#pragma unroll
  for (int r = 0; r < kEpMaxRanks; ++r) c[r] = 0;
  for (int i = i0; i < i1; ++i) {
    int lid;
    float g;
    const int r = pair_dest(p, i, lid, g, true);
#pragma unroll
    for (int q = 0; q < kEpMaxRanks; ++q) c[q] += (q == r) ? 1 : 0;
  }
#pragma unroll
  for (int r = 0; r < kEpMaxRanks; ++r) s_cnt[r][tid] = c[r];
  __syncthreads();
  // warp r: exclusive scan of rank r's counts over the 1024 threads (lane
  // holds 32 consecutive entries)
  if (warp < p.R) {
    int* row = s_cnt[warp];
    int v[32], sum = 0;
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      v[q] = row[lane * 32 + q];
      sum += v[q];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    int run = incl - sum;
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      row[lane * 32 + q] = run;
      run += v[q];
    }
    if (lane == 31) s_base[warp] = incl;  // rank total, turned into bases below
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int r = 0; r < p.R; ++r) {
      const int n = s_base[r];
      p.send_counts[r] = n;
      s_base[r] = acc;
      acc += n;
    }
  }
  __syncthreads();
  int next[kEpMaxRanks];
#pragma unroll
  for (int r = 0; r < kEpMaxRanks; ++r) next[r] = (r < p.R) ? s_base[r] + s_cnt[r][tid] : 0;
  const int slots = p.k + p.S;
  for (int i = i0; i < i1; ++i) {
    int lid = 0;
    float g = 0.f;
    const int r = pair_dest(p, i, lid, g, false);
    int pos = -1;
#pragma unroll
    for (int q = 0; q < kEpMaxRanks; ++q)
      if (q == r) pos = next[q]++;
    p.pair_pos[i] = pos;
    if (pos >= 0) {
      p.send_ids[pos] = lid;
      p.send_gates[pos] = g;
      p.send_token[pos] = i / slots;
    }
  }
}

__global__ void __launch_bounds__(256) k_ep_gather(const uint16_t* x, const int32_t* send_token,
                                                   const int32_t* send_counts, int R, int d, long long P,
                                                   uint16_t* send_x) {
  long long n = 0;
  for (int r = 0; r < R; ++r) n += send_counts[r];
  const int vpr = d / 8;
  const long long total = n * vpr;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = i / vpr;
    const int v = static_cast<int>(i % vpr);
    const int t = send_token[row];
    reinterpret_cast<uint4*>(send_x + row * d)[v] = __ldg(reinterpret_cast<const uint4*>(x + static_cast<long long>(t) * d) + v);
  }
}

__global__ void __launch_bounds__(256) k_ep_combine(const uint16_t* y, const int32_t* pair_pos, int T, int slots,
                                                    int d, const uint16_t* residual, uint16_t* out) {
  const int vpr = d / 8;
  const long long total = static_cast<long long>(T) * vpr;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i / vpr), v = static_cast<int>(i % vpr);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < slots; ++j) {
      const int pos = pair_pos[t * slots + j];
      if (pos < 0) continue;
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(y + static_cast<long long>(pos) * d) + v);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[2 * q] += __uint_as_float(ws[q] << 16);
        acc[2 * q + 1] += __uint_as_float(ws[q] & 0xFFFF0000u);
      }
    }
    if (residual != nullptr) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(residual + static_cast<long long>(t) * d) + v);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[2 * q] += __uint_as_float(ws[q] << 16);
        acc[2 * q + 1] += __uint_as_float(ws[q] & 0xFFFF0000u);
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
      o[q] = *reinterpret_cast<const uint32_t*>(&b);
    }
    reinterpret_cast<uint4*>(out + static_cast<long long>(t) * d)[v] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

bool al16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }
bool al4(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 3u) == 0; }

int grid_for(long long work) {
  long long b = (work + 255) / 256;
  if (b > 148LL * 8) b = 148LL * 8;
  return static_cast<int>(b < 1 ? 1 : b);
}

}  // namespace
}  // namespace flint

using namespace flint;

extern "C" int flint_ep_dispatch(const int32_t* topk_ids, const float* topk_weights, int32_t T, int32_t top_k,
                                 int32_t n_shared, int32_t n_experts, int32_t n_ranks, int32_t rank,
                                 const uint16_t* x, int32_t d, uint16_t* send_x, int32_t* send_ids,
                                 float* send_gates, int32_t* send_token, int32_t* send_counts, int32_t* pair_pos,
                                 int32_t* status, void* stream) {
  if (T < 0 || top_k < 1 || top_k > kEpMaxSlots - 1 || n_shared < 0 || n_shared > 1 || n_experts < 1 ||
      n_ranks < 1 || rank < 0 || rank >= n_ranks || d < 8 || d % 8 != 0)
    return flint_fail_external(FLINT_ERR_INVALID_ARG, "flint_ep_dispatch: bad sizes");
  if (n_ranks > kEpMaxRanks || n_experts % n_ranks != 0)
    return flint_fail_external(FLINT_ERR_UNSUPPORTED_SHAPE,
                               "flint_ep_dispatch: 1..8 ranks, n_experts a multiple of n_ranks");
  if (static_cast<long long>(T) * (top_k + n_shared) > (1LL << 22))
    return flint_fail_external(FLINT_ERR_UNSUPPORTED_SHAPE, "flint_ep_dispatch: at most 4M pairs");
  if (!send_counts) return flint_fail_external(FLINT_ERR_INVALID_ARG, "flint_ep_dispatch: NULL pointer");
  if (T > 0 && (!topk_ids || !topk_weights || !x || !send_x || !send_ids || !send_gates || !send_token ||
                !pair_pos))
    return flint_fail_external(FLINT_ERR_INVALID_ARG, "flint_ep_dispatch: NULL pointer");
  if (!al16(x) || !al16(send_x) || !al4(topk_ids) || !al4(topk_weights) || !al4(send_ids) || !al4(send_gates) ||
      !al4(send_token) || !al4(send_counts) || !al4(pair_pos))
    return flint_fail_external(FLINT_ERR_MISALIGNED, "flint_ep_dispatch: misaligned pointer");
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  PlanParams p{};
  p.ids = topk_ids;
  p.gates = topk_weights;
  p.send_ids = send_ids;
  p.send_gates = send_gates;
  p.send_token = send_token;
  p.send_counts = send_counts;
  p.pair_pos = pair_pos;
  p.status = status;
  p.T = T;
  p.k = top_k;
  p.S = n_shared;
  p.E = n_experts;
  p.R = n_ranks;
  p.rank = rank;
  k_ep_plan<<<1, kEpThreads, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return flint_fail_external(FLINT_ERR_CUDA, cudaGetErrorString(e));
  const long long P = static_cast<long long>(T) * (top_k + n_shared);
  if (P > 0) {
    k_ep_gather<<<grid_for(P * (d / 8)), 256, 0, st>>>(x, send_token, send_counts, n_ranks, d, P, send_x);
    e = cudaGetLastError();
    if (e != cudaSuccess) return flint_fail_external(FLINT_ERR_CUDA, cudaGetErrorString(e));
  }
  return FLINT_OK;
}

extern "C" int flint_ep_combine(const uint16_t* y, const int32_t* pair_pos, int32_t T, int32_t slots, int32_t d,
                                const uint16_t* residual, uint16_t* out, void* stream) {
  if (T < 0 || slots < 1 || slots > kEpMaxSlots || d < 8 || d % 8 != 0)
    return flint_fail_external(FLINT_ERR_INVALID_ARG, "flint_ep_combine: bad sizes");
  if (T == 0) return FLINT_OK;
  if (!y || !pair_pos || !out) return flint_fail_external(FLINT_ERR_INVALID_ARG, "flint_ep_combine: NULL pointer");
  if (!al16(y) || !al16(out) || (residual && !al16(residual)) || !al4(pair_pos))
    return flint_fail_external(FLINT_ERR_MISALIGNED, "flint_ep_combine: misaligned pointer");
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  k_ep_combine<<<grid_for(static_cast<long long>(T) * (d / 8)), 256, 0, st>>>(y, pair_pos, T, slots, d, residual,
                                                                             out);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return flint_fail_external(FLINT_ERR_CUDA, cudaGetErrorString(e));
  return FLINT_OK;
}
