// gemv.cuh -- shared pieces of the small-batch layer path: parameters, the
// routing descriptor, top-k by warp shuffles, token grouping, lane maps of the
// gate/up and down GEMVs, and warp reductions.
#pragma once

#include "common.cuh"

namespace flint {

constexpr int kMaxGemvTokens = 32;   // tokens per call on this path
constexpr int kMaxExperts = 512;
constexpr int kMaxTopK = 8;
constexpr int kMaxPairs = kMaxGemvTokens * kMaxTopK;
constexpr int kMaxStages = 8;
constexpr float kRmsEps = 1e-6f;

// Routing result published once per call by the router kernel's last CTA:
// active experts (routed in ascending id order, then the shared expert), the
// (token << 8 | slot) pairs of each in ascending token order, and per-token
// activation scales.
struct alignas(16) RouteDesc {
  int n_routed;                                     // routed experts in use
  int n_active;                                     // + shared experts
  int act[kMaxExperts + 1];                         // expert id per active slot
  int off[kMaxExperts + 2];                         // pair offsets per active slot
  unsigned short pair[kMaxPairs + kMaxGemvTokens];  // (token << 8) | slot
  float sigma[kMaxGemvTokens];                      // power-of-two f16 staging scale
  float irms[kMaxGemvTokens];                       // 1/rms(x) with input norm, else 1
};

// Everything a layer kernel needs; passed by value.
struct LayerParams {
  const uint16_t* x;         // [T][d] bf16
  const uint16_t* wr;        // [E][d] bf16
  const uint8_t* codes;      // packed E2M1 codes
  const uint8_t* scales;     // packed E4M3 block scales
  const float* tscale;       // [E+S][3]
  const uint16_t* residual;  // [T][d] bf16 or null
  uint16_t* out;             // [T][d] bf16
  int* status;               // workspace status word
  unsigned* counter;         // control block word 1: router arrival counter (self-resetting);
                             // word 2: launch generation of the persistent kernel
  RouteDesc* desc;           // routing descriptor (workspace)
  float* logits;             // [T][E]
  unsigned long long* tlogits;  // [8 tokens][replicas][E] tagged logits of the persistent kernel
  int* ids;                  // [T][k]
  float* gates;              // [T][k]
  float* h;                  // [T*(k+S)][I] fp32 SwiGLU intermediates
  unsigned long long* htag;  // [8*(k+S)][I] tagged h of the persistent kernel
  int* ids_out;              // optional public copy
  float* gates_out;          // optional public copy
  long long cpe;             // code bytes per expert (3*I*d/2)
  long long spe;             // scale bytes per expert (3*I*d/16)
  int T, d, I, E, k, S;
  int input_norm;            // 1: x / rms(x) feeds the router and the experts
  int x_in_smem;             // gate/up kernel stages x in shared memory
  int down_nb;               // output rows per down-kernel CTA
  int down_rb;               // rows per down work item
  int h_in_smem;             // down kernel stages every h row in shared memory
  int ns_gateup, ns_down;    // ring depths (stages per warp)
  int tc_lt;                 // tensor-core variant of the layer kernel: K-part sum slots per CTA
  int stage_gateup, stage_down;  // stage bytes
};

// ----------------------------------------------------------------- reductions
// Transposed butterfly reduction over aligned segments of SEG lanes. Each lane
// holds V partial values (V a power of two, V <= SEG); afterwards every lane
// holds the segment total of value index (lane_in_segment >> (log2 SEG - log2 V)).
// Costs V-1 + log2(SEG/V) shuffles instead of V*log2(SEG).
template <int O, int N>
struct XReduce {
  __device__ static __forceinline__ void run(float* v, int lane) {
    if constexpr (O == 0) {
      return;
    } else if constexpr (N > 1) {
      const bool up = (lane & O) != 0;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        const float send = up ? v[i] : v[i + N / 2];
        const float keep = up ? v[i + N / 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
      }
      XReduce<O / 2, N / 2>::run(v, lane);
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], O);
      XReduce<O / 2, 1>::run(v, lane);
    }
  }
};

template <int SEG, int V>
__device__ __forceinline__ float xreduce(float* v, int lane) {
  static_assert(V >= 1 && V <= SEG && (V & (V - 1)) == 0, "V must be a power of two <= SEG");
  XReduce<SEG / 2, V>::run(v, lane);
  return v[0];
}

__host__ __device__ constexpr int ilog2(int v) { return v <= 1 ? 0 : 1 + ilog2(v / 2); }

// ----------------------------------------------------------------- routing
// One warp, one token: top-k (k <= 8) of E <= 32*NE logits by k rounds of a
// warp-wide argmax. Each lane keeps its NE order-preserving 32-bit logit codes
// (larger logit = larger code, -0 == +0) and its current best; a round takes
// the warp maximum of the codes with redux.sync, then among the lanes holding
// that code the lowest expert index (a second redux over 0xFFFFFFFF - e), and
// the lane that owns the winner drops it. Gates are the renormalised softmax
// exp(l_j - l_max) / sum_sel exp(l_i - l_max). Lanes 0..k-1 write ids/gates.
__device__ __forceinline__ uint32_t route_code(float v) {
  if (v == 0.f) v = 0.f;
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float route_code_value(uint32_t ord) {
  return __uint_as_float((ord & 0x80000000u) ? (ord & 0x7FFFFFFFu) : ~ord);
}

// Selection on codes already loaded (code 0 = absent). Each lane first sorts
// its NE candidates (code descending, then expert index ascending) with a
// bitonic network, so a round only compares the lanes' heads: redux.sync
// takes the largest head code, a second one the lowest expert index among the
// lanes holding it, and the winning lane shifts its list. Round r's winner is
// kept by lane r; the rounds are a rolled loop (this runs once per token and
// launch, so its code size matters more than its unrolled speed).
template <int NE>
__device__ __forceinline__ void topk_select(uint32_t (&code)[NE], int k, int* ids, float* gates, int lane) {
  int slot[NE];
#pragma unroll
  for (int i = 0; i < NE; ++i) slot[i] = i;
  // descending bitonic sort of (code, -slot)
#pragma unroll
  for (int size = 2; size <= NE; size <<= 1) {
#pragma unroll
    for (int stride = size / 2; stride > 0; stride >>= 1) {
#pragma unroll
      for (int i = 0; i < NE; ++i) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0;
          // a "comes first" when its code is larger, or equal with a lower slot
          const bool i_first = code[i] > code[j] || (code[i] == code[j] && slot[i] < slot[j]);
          if (i_first != desc) {
            const uint32_t tc = code[i];
            code[i] = code[j];
            code[j] = tc;
            const int ts = slot[i];
            slot[i] = slot[j];
            slot[j] = ts;
          }
        }
      }
    }
  }
  float my_val = 0.f, v0 = 0.f;
  int my_sel = 0;
#pragma unroll 1
  for (int r = 0; r < k; ++r) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, code[0]);
    const uint32_t w = __reduce_max_sync(0xffffffffu, code[0] == m ? 0xFFFFFFFFu - (lane + 32 * slot[0]) : 0u);
    const int e = static_cast<int>(0xFFFFFFFFu - w);
    if ((e & 31) == lane) {  // the winner drops its head
#pragma unroll
      for (int i = 0; i + 1 < NE; ++i) {
        code[i] = code[i + 1];
        slot[i] = slot[i + 1];
      }
      code[NE - 1] = 0u;
    }
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

template <int NE>
__device__ __forceinline__ void topk_warp(const float* lg, int E, int k, int* ids, float* gates, int lane) {
  uint32_t code[NE];
#pragma unroll
  for (int i = 0; i < NE; ++i) {
    const int e = lane + 32 * i;
    // code 0 marks "absent"; a finite logit's code is never 0
    code[i] = (e < E) ? max(route_code(__ldcg(lg + e)), 1u) : 0u;
  }
  topk_select<NE>(code, k, ids, gates, lane);
}

__device__ __forceinline__ void topk_token(const float* lg, int E, int k, int* ids, float* gates, int lane) {
  if (E <= 256)
    topk_warp<8>(lg, E, k, ids, gates, lane);
  else
    topk_warp<kMaxExperts / 32>(lg, E, k, ids, gates, lane);
}

// Tagged logits: each is one 64-bit word (tag << 32 | float bits), stored with a
// single relaxed 64-bit store, so a reader that sees the current tag also sees
// that logit. Reading every logit of a token with the current tag is the
// producer/consumer handshake: no fence or counter is needed.
__device__ __forceinline__ void st_tagged(unsigned long long* p, uint32_t tag, float v) {
  const unsigned long long w = (static_cast<unsigned long long>(tag) << 32) | __float_as_uint(v);
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ unsigned long long ld_tagged(const unsigned long long* p) {
  unsigned long long w;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
  return w;
}

// One warp, one token: waits (bounded) until all E logits carry `tag`, then
// selects as topk_warp. Returns false (and records FLINT_DEVCHECK_WAIT) if the
// wait gave up.
template <int NE>
__device__ __forceinline__ bool topk_warp_tagged(const unsigned long long* lg, int E, int k, uint32_t tag, int* ids,
                                                 float* gates, int lane, int* status) {
  uint32_t code[NE];
  unsigned pending = 0;
#pragma unroll
  for (int i = 0; i < NE; ++i)
    if (lane + 32 * i < E) pending |= 1u << i;
  const long long t0 = clock64();
  bool ok = true;
  for (;;) {
    unsigned long long w[NE];  // all loads issued before any is inspected
#pragma unroll
    for (int i = 0; i < NE; ++i) w[i] = (pending & (1u << i)) ? ld_tagged(lg + lane + 32 * i) : 0ull;
#pragma unroll
    for (int i = 0; i < NE; ++i) {
      if ((pending & (1u << i)) && static_cast<uint32_t>(w[i] >> 32) == tag) {
        pending &= ~(1u << i);
        code[i] = max(route_code(__uint_as_float(static_cast<uint32_t>(w[i]))), 1u);
      }
    }
    if (__all_sync(0xffffffffu, pending == 0)) break;
    if (clock64() - t0 > kWaitCycles) {
      ok = false;
      break;
    }
  }
  if (!ok) {
    if (lane == 0) atomicOr(status, FLINT_DEVCHECK_WAIT);
    return false;
  }
#pragma unroll
  for (int i = 0; i < NE; ++i)
    if (lane + 32 * i >= E) code[i] = 0u;
  topk_select<NE>(code, k, ids, gates, lane);
  return true;
}

// Token grouping built by a whole CTA from ids [T][k] (T <= 32): active
// experts in ascending id order (then the shared experts, with every token in
// slot k+s), and for each its (token, slot) pairs in ascending token order.
struct Grouping {
  int n_active;
  int n_routed;
  int act[kMaxExperts + 1];
  int off[kMaxExperts + 2];
  unsigned short pair[kMaxPairs + kMaxGemvTokens];
  int ecount[kMaxExperts];   // scratch: per-expert count, then offset
  unsigned emask[kMaxExperts];  // scratch: per-expert token bitmask
};

inline __device__ void build_grouping(Grouping& g, const int* ids, int T, int k, int E, int S, int* status) {
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) {
    g.ecount[e] = 0;
    g.emask[e] = 0u;
  }
  __syncthreads();
  for (int i = tid; i < T * k; i += blockDim.x) {
    const int e = ids[i];
    if (e < 0 || e >= E) {
      atomicOr(status, FLINT_DEVCHECK_EXPERT_ID);
      continue;
    }
    atomicAdd(&g.ecount[e], 1);
    atomicOr(&g.emask[e], 1u << (i / k));
  }
  __syncthreads();
  if (tid < 32) {
    const int per = (E + 31) / 32;
    const int e0 = tid * per;
    int cnt = 0, act = 0;
    for (int i = 0; i < per; ++i) {
      const int e = e0 + i;
      if (e < E) {
        cnt += g.ecount[e];
        act += g.ecount[e] > 0;
      }
    }
    int cnt_ex = cnt, act_ex = act;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, cnt_ex, o);
      const int b = __shfl_up_sync(0xffffffffu, act_ex, o);
      if (tid >= o) {
        cnt_ex += a;
        act_ex += b;
      }
    }
    cnt_ex -= cnt;
    act_ex -= act;
    for (int i = 0; i < per; ++i) {
      const int e = e0 + i;
      if (e < E) {
        const int c = g.ecount[e];
        if (c > 0) {
          g.act[act_ex] = e;
          g.off[act_ex] = cnt_ex;
          ++act_ex;
        }
        g.ecount[e] = cnt_ex;
        cnt_ex += c;
      }
    }
    if (tid == 31) {
      g.n_routed = act_ex;
      int na = act_ex, total = cnt_ex;
      for (int s = 0; s < S; ++s) {
        g.act[na] = E + s;
        g.off[na] = total;
        total += T;
        ++na;
      }
      g.off[na] = total;
      g.n_active = na;
    }
  }
  __syncthreads();
  for (int i = tid; i < T * k; i += blockDim.x) {
    const int e = ids[i];
    if (e < 0 || e >= E) continue;
    const int t = i / k, j = i % k;
    const int pos = g.ecount[e] + __popc(g.emask[e] & ((1u << t) - 1u));
    g.pair[pos] = static_cast<unsigned short>((t << 8) | j);
  }
  for (int i = tid; i < S * T; i += blockDim.x) {
    const int s = i / T, t = i % T;
    g.pair[g.off[g.n_routed + s] + t] = static_cast<unsigned short>((t << 8) | (k + s));
  }
  __syncthreads();
}

// Warp-synchronous token grouping for T*k <= 64 pairs: a bitonic sort of the
// keys (expert << 16 | token << 8 | slot), two per lane, then run boundaries
// by ballot. Writes the same descriptor fields as build_grouping.
inline __device__ void warp_grouping(const int* ids, int T, int k, int E, int S, RouteDesc* d, int lane,
                              int* status) {
  const int n = T * k;
  uint32_t key[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i = 2 * lane + h;
    uint32_t kv = 0xFFFFFFFFu;
    if (i < n) {
      int e = ids[i];
      if (e < 0 || e >= E) {  // cannot come from top-k; keep indexing in bounds
        atomicOr(status, FLINT_DEVCHECK_EXPERT_ID);
        e = 0;
      }
      kv = (static_cast<uint32_t>(e) << 16) | (static_cast<uint32_t>(i / k) << 8) | static_cast<uint32_t>(i % k);
    }
    key[h] = kv;
  }
  // bitonic sort of 64 keys; element index i = 2*lane + h
#pragma unroll
  for (int size = 2; size <= 64; size <<= 1) {
#pragma unroll
    for (int stride = size / 2; stride > 0; stride >>= 1) {
      if (stride == 1) {
        const bool asc = ((2 * lane) & size) == 0;
        const uint32_t lo = min(key[0], key[1]), hi = max(key[0], key[1]);
        key[0] = asc ? lo : hi;
        key[1] = asc ? hi : lo;
      } else {
        const int lstride = stride / 2;  // partner lane distance
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int i = 2 * lane + h;
          const uint32_t other = __shfl_xor_sync(0xffffffffu, key[h], lstride);
          const bool asc = (i & size) == 0;
          const bool lower = (i & stride) == 0;
          key[h] = (asc == lower) ? min(key[h], other) : max(key[h], other);
        }
      }
    }
  }
  // run boundaries (new expert) and their ranks
  const uint32_t prev_b = __shfl_up_sync(0xffffffffu, key[1], 1);
  const bool valid0 = (2 * lane) < n, valid1 = (2 * lane + 1) < n;
  const bool b0 = valid0 && (lane == 0 || (key[0] >> 16) != (prev_b >> 16));
  const bool b1 = valid1 && ((key[1] >> 16) != (key[0] >> 16));
  const uint32_t m0 = __ballot_sync(0xffffffffu, b0), m1 = __ballot_sync(0xffffffffu, b1);
  const uint32_t below = (1u << lane) - 1u;
  const int r0 = __popc(m0 & below) + __popc(m1 & below);  // boundaries before element 2*lane
  const int r1 = r0 + (b0 ? 1 : 0);
  const int U = __popc(m0) + __popc(m1);
  if (b0) {
    d->act[r0] = static_cast<int>(key[0] >> 16);
    d->off[r0] = 2 * lane;
  }
  if (b1) {
    d->act[r1] = static_cast<int>(key[1] >> 16);
    d->off[r1] = 2 * lane + 1;
  }
  if (valid0) d->pair[2 * lane] = static_cast<unsigned short>(key[0] & 0xFFFFu);
  if (valid1) d->pair[2 * lane + 1] = static_cast<unsigned short>(key[1] & 0xFFFFu);
  for (int i = lane; i < S * T; i += 32) {
    const int s = i / T, t = i % T;
    d->pair[n + i] = static_cast<unsigned short>((t << 8) | (k + s));
  }
  if (lane == 0) {
    for (int s = 0; s < S; ++s) {
      d->act[U + s] = E + s;
      d->off[U + s] = n + s * T;
    }
    d->off[U + S] = n + S * T;
    d->n_routed = U;
    d->n_active = U + S;
  }
}

// Token grouping by a whole CTA (blockDim.x >= E/2, a multiple of 32) for
// T <= 128 tokens, through a token mask per expert (two 64-bit words): pair
// i = t*k + j sets bit t of its expert's mask (a token picks an expert at most
// once), so a pair's place among its expert's pairs (token order) is the
// popcount of the mask below bit t; exclusive scans over the experts give the
// active list (ascending id) and the offsets. Shared experts follow, with
// every token in slot k+s. `scratch`: 20*E bytes of shared memory, 8-byte
// aligned. Writes act/off/pair and the two counts.
template <typename PairT>
__device__ void cta_grouping(const int* ids, int T, int k, int E, int S, int* act, int* off, PairT* pair,
                             int* n_routed, int* n_active, uint8_t* scratch, int* status) {
  __shared__ int s_tot[2][32];
  unsigned long long* emask = reinterpret_cast<unsigned long long*>(scratch);  // [E][2]
  int* eoff = reinterpret_cast<int*>(scratch + 16 * static_cast<size_t>(E));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5, n = T * k;
  for (int i = tid; i < 2 * E; i += blockDim.x) emask[i] = 0ull;
  __syncthreads();
  for (int i = tid; i < n; i += blockDim.x) {
    const int e = ids[i], t = i / k;
    if (e < 0 || e >= E) {
      atomicOr(status, FLINT_DEVCHECK_EXPERT_ID);
      continue;
    }
    atomicOr(&emask[2 * e + (t >> 6)], 1ull << (t & 63));
  }
  __syncthreads();
  // thread owns experts 2*tid and 2*tid+1
  const int e0 = 2 * tid, e1 = 2 * tid + 1;
  const int c0 = e0 < E ? __popcll(emask[2 * e0]) + __popcll(emask[2 * e0 + 1]) : 0;
  const int c1 = e1 < E ? __popcll(emask[2 * e1]) + __popcll(emask[2 * e1 + 1]) : 0;
  const int f0 = c0 > 0, f1 = c1 > 0;
  int ic = c0 + c1, jf = f0 + f1;  // inclusive scans over the block
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int vc = __shfl_up_sync(0xffffffffu, ic, o), vf = __shfl_up_sync(0xffffffffu, jf, o);
    if (lane >= o) {
      ic += vc;
      jf += vf;
    }
  }
  if (lane == 31) {
    s_tot[0][warp] = ic;
    s_tot[1][warp] = jf;
  }
  __syncthreads();
  if (warp == 0) {
    int wc = lane < nw ? s_tot[0][lane] : 0, wf = lane < nw ? s_tot[1][lane] : 0;
    const int xc = wc, xf = wf;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int vc = __shfl_up_sync(0xffffffffu, wc, o), vf = __shfl_up_sync(0xffffffffu, wf, o);
      if (lane >= o) {
        wc += vc;
        wf += vf;
      }
    }
    __syncwarp();
    if (lane < nw) {
      s_tot[0][lane] = wc - xc;  // exclusive prefix of the warp totals
      s_tot[1][lane] = wf - xf;
    }
    if (lane == nw - 1) {
      *n_routed = wf;
      *n_active = wf + S;
      for (int s = 0; s < S; ++s) {
        act[wf + s] = E + s;
        off[wf + s] = wc + s * T;
      }
      off[wf + S] = wc + S * T;
    }
  }
  __syncthreads();
  const int base_c = ic - (c0 + c1) + s_tot[0][warp], base_f = jf - (f0 + f1) + s_tot[1][warp];
  if (f0) {
    act[base_f] = e0;
    off[base_f] = base_c;
    eoff[e0] = base_c;
  }
  if (f1) {
    act[base_f + f0] = e1;
    off[base_f + f0] = base_c + c0;
    eoff[e1] = base_c + c0;
  }
  __syncthreads();
  for (int i = tid; i < n; i += blockDim.x) {
    const int e = ids[i];
    if (e < 0 || e >= E) continue;
    const int t = i / k;
    const unsigned long long lo = emask[2 * e], hi = emask[2 * e + 1];
    const int below = t < 64 ? __popcll(lo & ((1ull << t) - 1ull))
                             : __popcll(lo) + __popcll(hi & ((1ull << (t - 64)) - 1ull));
    pair[eoff[e] + below] = static_cast<PairT>((t << 8) | (i % k));
  }
  const int nr = off[*n_routed];  // the shared experts' pairs follow the routed ones
  for (int i = tid; i < S * T; i += blockDim.x) {
    const int s = i / T, t = i % T;
    pair[nr + i] = static_cast<PairT>((t << 8) | (k + s));
  }
  __syncthreads();
}

// ----------------------------------------------------------------- gate/up lane map
// A unit is [gate row u | up row u] (D columns each). Lane's j-th 16-byte code
// vector covers columns 32*cb .. 32*cb+31 of row r, with x column block xi.
template <int D>
struct GateUpMap {
  static constexpr int VR = D / 32;                    // 16-byte code vectors per row
  static constexpr int NVU = D / 512;                  // vectors per lane per unit
  static constexpr int XV = (VR >= 32) ? VR / 32 : 1;  // x column blocks per lane
  static constexpr int XS = XV * 16;                   // f16x2 registers per token
  static constexpr int TGMAX = (D == 4096) ? 1 : 2;     // tokens per pass
  static constexpr int CU = (D <= 1024) ? 4 : (D == 2048 ? 2 : 1);  // units per chunk
  static constexpr int UNIT_CODE = D;
  static constexpr int UNIT_SCALE = D / 8;
  static constexpr int UNIT_BYTES = UNIT_CODE + UNIT_SCALE;
  __device__ static __forceinline__ int xblock(int lane, int xi) {
    return (VR >= 32) ? lane + 32 * xi : (lane & 15);
  }
  __device__ static __forceinline__ void vec(int lane, int j, int& code_off, int& scale_off, int& row,
                                             int& xi) {
    int cb;
    if constexpr (VR >= 32) {
      row = j / XV;
      xi = j % XV;
      cb = lane + 32 * xi;
    } else {
      row = lane >> 4;
      xi = 0;
      cb = lane & 15;
    }
    code_off = row * (D / 2) + cb * 16;
    scale_off = row * (D / 16) + cb * 2;
  }
};

// bf16 words -> f16x2 scaled by sg (element 2i in the low half).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_scaled(uint32_t w, float sg) {
  return pack_f16x2(bf16_bits_to_f32(w & 0xFFFFu) * sg, __uint_as_float(w & 0xFFFF0000u) * sg);
}

}  // namespace flint
