// flint_oracle.cpp -- plain fp64 CPU oracle of one Flint MoE layer's decode step.
//
// TEST INFRASTRUCTURE (see flint_oracle.h): only tests/, __graft_entry__.smoke()
// and bench.py's CPU baseline use it; the CUDA library never does.
//
// Everything here is written for a reader checking it against the definitions by
// eye: no blocking, fusion or reordering beyond what each definition states.
// Build with -ffp-contract=off (the quantiser's fp32 steps must not be fused).

#include "flint_oracle.h"

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <thread>
#include <vector>

namespace {

double bf16_bits_to_double(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

// silu(g) = g * sigmoid(g) = g / (1 + e^-g)   (SwiGLU gate activation)
double silu(double g) { return g / (1.0 + std::exp(-g)); }

}  // namespace

extern "C" {

// ---------------------------------------------------------------------------
// Element codecs. OCP Microscaling (MX) v1.0 element formats.
// ---------------------------------------------------------------------------

// FP4 E2M1: sign = bit 3, exponent = bits 2..1 (bias 1), mantissa = bit 0.
// Exponent 0 is subnormal: value = m * 0.5. Otherwise 2^(e-1) * (1 + m/2).
double oracle_e2m1_decode(uint8_t code) {
  const int s = (code >> 3) & 1;
  const int e = (code >> 1) & 3;
  const int m = code & 1;
  const double mag = (e == 0) ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, e - 1);
  return s ? -mag : mag;
}

// FP8 E4M3 ("fn" variant): sign = bit 7, exponent = bits 6..3 (bias 7),
// mantissa = bits 2..0. Exponent 0 is subnormal: (m/8) * 2^-6. Otherwise
// 2^(e-7) * (1 + m/8). S.1111.111 is NaN; there are no infinities.
double oracle_e4m3_decode(uint8_t code) {
  const int s = (code >> 7) & 1;
  const int e = (code >> 3) & 15;
  const int m = code & 7;
  if (e == 15 && m == 7) return std::nan("");
  const double mag = (e == 0) ? std::ldexp(m / 8.0, -6) : std::ldexp(1.0 + m / 8.0, e - 7);
  return s ? -mag : mag;
}

// Round |v| to the E2M1 grid: spacing 0.5 below 2 (subnormals included),
// 1 in [2,4), 2 in [4,6]; ties go to the even integer multiple of the spacing,
// which is the code with mantissa bit 0. Anything >= 6 saturates to 6.
uint8_t oracle_e2m1_encode(float v) {
  const uint8_t sign = std::signbit(v) ? 0x8 : 0x0;
  const double a = std::fabs(static_cast<double>(v));
  if (std::isnan(v)) return sign | 0x7;  // outside the quantiser's domain
  double q;
  if (a >= 6.0) {
    q = 6.0;
  } else {
    const double spacing = (a < 2.0) ? 0.5 : (a < 4.0 ? 1.0 : 2.0);
    q = std::nearbyint(a / spacing) * spacing;  // default rounding mode: ties to even
    if (q > 6.0) q = 6.0;
  }
  for (uint8_t c = 0; c < 8; ++c)
    if (oracle_e2m1_decode(c) == q) return sign | c;
  return sign | 0x7;  // unreachable
}

// Round |v| to the E4M3 grid: in binade [2^E, 2^(E+1)) (E >= -6; below 2^-6 the
// subnormal spacing 2^-9 applies) the spacing is 2^(E-3); ties to even.
// Values at or above the largest finite value 448 saturate to 448.
uint8_t oracle_e4m3_encode(float v) {
  const uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
  const double a = std::fabs(static_cast<double>(v));
  if (std::isnan(v)) return sign | 0x7F;
  double q;
  if (a >= 448.0) {
    q = 448.0;
  } else {
    int E = -6;
    if (a >= std::ldexp(1.0, -6)) {
      int ex;
      std::frexp(a, &ex);  // a = f * 2^ex, f in [0.5, 1)
      E = ex - 1;
    }
    const double spacing = std::ldexp(1.0, E - 3);
    q = std::nearbyint(a / spacing) * spacing;
    if (q > 448.0) q = 448.0;
  }
  for (int c = 0; c <= 0x7E; ++c)
    if (oracle_e4m3_decode(static_cast<uint8_t>(c)) == q) return sign | static_cast<uint8_t>(c);
  return sign | 0x7E;  // unreachable
}

// bf16 keeps 8 significant bits; normal binades 2^-126..2^127, subnormal
// spacing 2^-133. Round to nearest, ties to even.
uint16_t oracle_bf16_from_double(double v) {
  if (std::isnan(v)) return 0x7FC0;
  const uint16_t sign = std::signbit(v) ? 0x8000 : 0x0000;
  const double a = std::fabs(v);
  if (a == 0.0) return sign;
  int ex;
  std::frexp(a, &ex);
  int E = ex - 1;  // a in [2^E, 2^(E+1))
  if (E < -126) E = -126;
  const double spacing = std::ldexp(1.0, E - 7);
  const double q = std::nearbyint(a / spacing) * spacing;
  const double max_finite = std::ldexp(255.0, 127 - 7);  // (2 - 2^-7) * 2^127
  if (q > max_finite) return sign | 0x7F80;              // rounds past the top: inf
  const float f = static_cast<float>(q);                  // exact: q has <= 8 bits
  uint32_t u;
  std::memcpy(&u, &f, sizeof u);
  return sign | static_cast<uint16_t>((u >> 16) & 0x7FFF);
}

double oracle_bf16_to_double(uint16_t bits) { return bf16_bits_to_double(bits); }

// ---------------------------------------------------------------------------
// NVFP4 quantiser (fp32 recipe; see header).
// ---------------------------------------------------------------------------
int oracle_quantize_nvfp4(const float* w, int32_t rows, int32_t cols, uint8_t* codes,
                          uint8_t* scales, float* tensor_scale) {
  if (rows <= 0 || cols <= 0 || cols % 16 != 0) return -1;
  const size_t n = static_cast<size_t>(rows) * cols;
  float amax = 0.0f;
  for (size_t i = 0; i < n; ++i) {
    if (!std::isfinite(w[i])) return -1;
    const float a = std::fabs(w[i]);
    if (a > amax) amax = a;
  }
  return oracle_quantize_nvfp4_rows(w, rows, cols, amax, codes, scales, tensor_scale);
}

int oracle_quantize_nvfp4_rows(const float* w, int32_t rows, int32_t cols, float amax, uint8_t* codes,
                               uint8_t* scales, float* tensor_scale) {
  if (rows <= 0 || cols <= 0 || cols % 16 != 0 || !(amax >= 0.0f) || !std::isfinite(amax)) return -1;
  for (size_t i = 0; i < static_cast<size_t>(rows) * cols; ++i)
    if (!std::isfinite(w[i]) || std::fabs(w[i]) > amax) return -1;
  // 2688 = 6 (largest E2M1) * 448 (largest E4M3)
  const float s_t = (amax > 0.0f) ? amax / 2688.0f : 1.0f;
  *tensor_scale = s_t;
  const int nblocks = cols / 16;
  for (int r = 0; r < rows; ++r) {
    for (int b = 0; b < nblocks; ++b) {
      const float* blk = w + static_cast<size_t>(r) * cols + 16 * b;
      float amax_b = 0.0f;
      for (int i = 0; i < 16; ++i) amax_b = std::max(amax_b, std::fabs(blk[i]));
      const float v = (amax_b / 6.0f) / s_t;
      const uint8_t sb = oracle_e4m3_encode(v);
      scales[static_cast<size_t>(r) * nblocks + b] = sb;
      const float denom = static_cast<float>(oracle_e4m3_decode(sb)) * s_t;
      for (int i = 0; i < 16; ++i) {
        const uint8_t q = (denom == 0.0f) ? 0 : oracle_e2m1_encode(blk[i] / denom);
        const int col = 16 * b + i;
        uint8_t& byte = codes[static_cast<size_t>(r) * (cols / 2) + col / 2];
        if (col % 2 == 0)
          byte = static_cast<uint8_t>((byte & 0xF0) | q);
        else
          byte = static_cast<uint8_t>((byte & 0x0F) | (q << 4));
      }
    }
  }
  return 0;
}

int oracle_decode_matrix(const oracle_matrix* m, double* out) {
  if (!m || !out) return -1;
  const int rows = m->rows, cols = m->cols;
  if (m->kind == 1) {
    if (!m->bf16) return -1;
    for (size_t i = 0; i < static_cast<size_t>(rows) * cols; ++i) out[i] = bf16_bits_to_double(m->bf16[i]);
    return 0;
  }
  if (!m->codes || !m->scales || cols % 16 != 0) return -1;
  const double s_t = static_cast<double>(m->tensor_scale);
  for (int r = 0; r < rows; ++r) {
    for (int c = 0; c < cols; ++c) {
      const uint8_t byte = m->codes[static_cast<size_t>(r) * (cols / 2) + c / 2];
      const uint8_t q = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);
      const uint8_t sb = m->scales[static_cast<size_t>(r) * (cols / 16) + c / 16];
      out[static_cast<size_t>(r) * cols + c] = oracle_e2m1_decode(q) * oracle_e4m3_decode(sb) * s_t;
    }
  }
  return 0;
}

// ---------------------------------------------------------------------------
// Packed layout (see header for the definition being restated).
// ---------------------------------------------------------------------------
int oracle_pack_layout(const oracle_matrix* mats, int32_t n_experts_total, int32_t d,
                       int32_t inter, uint8_t* packed_codes, uint8_t* packed_scales,
                       float* tensor_scales) {
  if (d % 32 != 0 || inter % 32 != 0) return -1;
  const size_t codes_per_expert = static_cast<size_t>(3) * inter * d / 2;
  const size_t scales_per_expert = static_cast<size_t>(3) * inter * d / 16;
  for (int e = 0; e < n_experts_total; ++e) {
    const oracle_matrix& g = mats[3 * e + 0];
    const oracle_matrix& u = mats[3 * e + 1];
    const oracle_matrix& dn = mats[3 * e + 2];
    uint8_t* ce = packed_codes + e * codes_per_expert;
    uint8_t* se = packed_scales + e * scales_per_expert;
    // gate/up units: unit i = [gate row i | up row i]
    for (int i = 0; i < inter; ++i) {
      std::memcpy(ce + static_cast<size_t>(i) * d, g.codes + static_cast<size_t>(i) * (d / 2), d / 2);
      std::memcpy(ce + static_cast<size_t>(i) * d + d / 2, u.codes + static_cast<size_t>(i) * (d / 2), d / 2);
      std::memcpy(se + static_cast<size_t>(i) * (d / 8), g.scales + static_cast<size_t>(i) * (d / 16), d / 16);
      std::memcpy(se + static_cast<size_t>(i) * (d / 8) + d / 16, u.scales + static_cast<size_t>(i) * (d / 16), d / 16);
    }
    // down rows follow
    uint8_t* cd = ce + static_cast<size_t>(inter) * d;
    uint8_t* sd = se + static_cast<size_t>(inter) * d / 8;
    for (int r = 0; r < d; ++r) {
      std::memcpy(cd + static_cast<size_t>(r) * (inter / 2), dn.codes + static_cast<size_t>(r) * (inter / 2), inter / 2);
      std::memcpy(sd + static_cast<size_t>(r) * (inter / 16), dn.scales + static_cast<size_t>(r) * (inter / 16), inter / 16);
    }
    tensor_scales[3 * e + 0] = g.tensor_scale;
    tensor_scales[3 * e + 1] = u.tensor_scale;
    tensor_scales[3 * e + 2] = dn.tensor_scale;
  }
  return 0;
}

int oracle_pack_layout_bf16(const oracle_matrix* mats, int32_t n_experts_total, int32_t d,
                            int32_t inter, uint16_t* packed) {
  const size_t per_expert = static_cast<size_t>(3) * inter * d;
  for (int e = 0; e < n_experts_total; ++e) {
    const oracle_matrix& g = mats[3 * e + 0];
    const oracle_matrix& u = mats[3 * e + 1];
    const oracle_matrix& dn = mats[3 * e + 2];
    uint16_t* pe = packed + e * per_expert;
    for (int i = 0; i < inter; ++i) {
      std::memcpy(pe + static_cast<size_t>(i) * 2 * d, g.bf16 + static_cast<size_t>(i) * d, d * 2);
      std::memcpy(pe + static_cast<size_t>(i) * 2 * d + d, u.bf16 + static_cast<size_t>(i) * d, d * 2);
    }
    uint16_t* pd = pe + static_cast<size_t>(2) * inter * d;
    std::memcpy(pd, dn.bf16, static_cast<size_t>(d) * inter * 2);
  }
  return 0;
}

// ---------------------------------------------------------------------------
// Routing: router GEMV, softmax over all experts, top-k, renormalise.
// ---------------------------------------------------------------------------
int oracle_router_logits(const uint16_t* x, int32_t T, const uint16_t* wr, int32_t d,
                         int32_t E, double* logits) {
  for (int t = 0; t < T; ++t)
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int j = 0; j < d; ++j)
        acc += bf16_bits_to_double(x[static_cast<size_t>(t) * d + j]) *
               bf16_bits_to_double(wr[static_cast<size_t>(e) * d + j]);
      logits[static_cast<size_t>(t) * E + e] = acc;
    }
  return 0;
}

int oracle_topk(const double* logits, int32_t T, int32_t E, int32_t k, int32_t* ids,
                double* gates, double* gap) {
  if (k < 1 || k > E) return -1;
  std::vector<int> order(E);
  std::vector<double> p(E);
  for (int t = 0; t < T; ++t) {
    const double* l = logits + static_cast<size_t>(t) * E;
    for (int e = 0; e < E; ++e)
      if (std::isnan(l[e])) return -1;
    for (int e = 0; e < E; ++e) order[e] = e;
    // larger logit first; equal logits (+0 and -0 compare equal) -> lower index first
    std::sort(order.begin(), order.end(), [&](int a, int b) {
      if (l[a] != l[b]) return l[a] > l[b];
      return a < b;
    });
    // full softmax over all E logits
    const double m = l[order[0]];
    double z = 0.0;
    for (int e = 0; e < E; ++e) {
      p[e] = std::exp(l[e] - m);
      z += p[e];
    }
    for (int e = 0; e < E; ++e) p[e] /= z;
    double sel = 0.0;
    for (int j = 0; j < k; ++j) sel += p[order[j]];
    for (int j = 0; j < k; ++j) {
      if (ids) ids[static_cast<size_t>(t) * k + j] = order[j];
      if (gates) gates[static_cast<size_t>(t) * k + j] = p[order[j]] / sel;
    }
    if (gap) gap[t] = (k < E) ? p[order[k - 1]] - p[order[k]] : INFINITY;
  }
  return 0;
}

// ---------------------------------------------------------------------------
// Experts.
// ---------------------------------------------------------------------------
namespace {

struct DecodedExpert {
  std::vector<double> wg, wu, wd;  // gate [I][d], up [I][d], down [d][I]
};

int decode_expert(const oracle_matrix* m3, int d, int inter, DecodedExpert* out) {
  out->wg.assign(static_cast<size_t>(inter) * d, 0.0);
  out->wu.assign(static_cast<size_t>(inter) * d, 0.0);
  out->wd.assign(static_cast<size_t>(d) * inter, 0.0);
  if (m3[0].rows != inter || m3[0].cols != d || m3[1].rows != inter || m3[1].cols != d ||
      m3[2].rows != d || m3[2].cols != inter)
    return -1;
  if (oracle_decode_matrix(&m3[0], out->wg.data())) return -1;
  if (oracle_decode_matrix(&m3[1], out->wu.data())) return -1;
  if (oracle_decode_matrix(&m3[2], out->wd.data())) return -1;
  return 0;
}

// y = W_d (silu(W_g x) * (W_u x)), all fp64.
void ffn_decoded(const DecodedExpert& w, int d, int inter, const double* x, double* y) {
  std::vector<double> h(inter);
  for (int i = 0; i < inter; ++i) {
    double g = 0.0, u = 0.0;
    for (int j = 0; j < d; ++j) {
      g += w.wg[static_cast<size_t>(i) * d + j] * x[j];
      u += w.wu[static_cast<size_t>(i) * d + j] * x[j];
    }
    h[i] = silu(g) * u;
  }
  for (int n = 0; n < d; ++n) {
    double acc = 0.0;
    for (int i = 0; i < inter; ++i) acc += w.wd[static_cast<size_t>(n) * inter + i] * h[i];
    y[n] = acc;
  }
}

}  // namespace

int oracle_expert_ffn(const oracle_matrix* mats, int32_t d, int32_t inter, const double* x,
                      double* y) {
  DecodedExpert w;
  if (decode_expert(mats, d, inter, &w)) return -1;
  ffn_decoded(w, d, inter, x, y);
  return 0;
}

int oracle_moe_forward(int32_t T, int32_t d, int32_t inter, int32_t E, int32_t k, int32_t S,
                       const uint16_t* x, const uint16_t* wr, const oracle_matrix* mats,
                       const uint16_t* residual, const int32_t* ids_override, int32_t input_norm,
                       int32_t n_threads,
                       int32_t* ids_out, double* gates_out, double* gap_out, double* logits_out,
                       double* out) {
  if (T < 0 || d <= 0 || inter <= 0 || E <= 0 || k < 1 || k > E || S < 0) return -1;
  if (T == 0) return 0;
  // 0. layer input: x, or x / rms(x) with input_norm
  std::vector<double> xd(static_cast<size_t>(T) * d);
  for (size_t i = 0; i < xd.size(); ++i) xd[i] = bf16_bits_to_double(x[i]);
  if (input_norm) {
    for (int t = 0; t < T; ++t) {
      double ms = 0.0;
      for (int j = 0; j < d; ++j) ms += xd[static_cast<size_t>(t) * d + j] * xd[static_cast<size_t>(t) * d + j];
      const double r = std::sqrt(ms / d + 1e-6);
      for (int j = 0; j < d; ++j) xd[static_cast<size_t>(t) * d + j] /= r;
    }
  }
  // 1. router logits and top-k gating
  std::vector<double> logits(static_cast<size_t>(T) * E);
  std::vector<double> wrd(static_cast<size_t>(E) * d);
  for (size_t i = 0; i < wrd.size(); ++i) wrd[i] = bf16_bits_to_double(wr[i]);
  for (int t = 0; t < T; ++t)
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int j = 0; j < d; ++j) acc += xd[static_cast<size_t>(t) * d + j] * wrd[static_cast<size_t>(e) * d + j];
      logits[static_cast<size_t>(t) * E + e] = acc;
    }
  std::vector<int32_t> ids(static_cast<size_t>(T) * k);
  std::vector<double> gates(static_cast<size_t>(T) * k), gap(T);
  if (oracle_topk(logits.data(), T, E, k, ids.data(), gates.data(), gap.data())) return -1;
  if (ids_override) {
    // forced ids: gates are those experts' softmax probabilities, renormalised
    for (int t = 0; t < T; ++t) {
      const double* l = logits.data() + static_cast<size_t>(t) * E;
      double m = l[0];
      for (int e = 1; e < E; ++e) m = std::max(m, l[e]);
      double sel = 0.0;
      for (int j = 0; j < k; ++j) {
        const int e = ids_override[static_cast<size_t>(t) * k + j];
        if (e < 0 || e >= E) return -1;
        sel += std::exp(l[e] - m);
      }
      for (int j = 0; j < k; ++j) {
        const int e = ids_override[static_cast<size_t>(t) * k + j];
        ids[static_cast<size_t>(t) * k + j] = e;
        gates[static_cast<size_t>(t) * k + j] = std::exp(l[e] - m) / sel;
      }
    }
  }
  // 2. every (token, slot) pair: slots 0..k-1 are the routed experts, k..k+S-1 the shared ones
  const int slots = k + S;
  std::vector<double> y(static_cast<size_t>(T) * slots * d, 0.0);
  // one job per expert in use: decode it once, run it for each token that selected it
  std::vector<std::vector<std::pair<int, int>>> users(E + S);
  for (int t = 0; t < T; ++t) {
    for (int j = 0; j < k; ++j) users[ids[static_cast<size_t>(t) * k + j]].push_back({t, j});
    for (int s = 0; s < S; ++s) users[E + s].push_back({t, k + s});
  }
  std::vector<int> jobs;
  for (int e = 0; e < E + S; ++e)
    if (!users[e].empty()) jobs.push_back(e);
  std::atomic<int> next{0};
  std::atomic<int> failed{0};
  auto worker = [&]() {
    DecodedExpert w;
    for (;;) {
      const int j = next.fetch_add(1);
      if (j >= static_cast<int>(jobs.size())) return;
      const int e = jobs[j];
      if (decode_expert(&mats[3 * e], d, inter, &w)) {
        failed = 1;
        return;
      }
      for (const auto& ts : users[e])
        ffn_decoded(w, d, inter, xd.data() + static_cast<size_t>(ts.first) * d,
                    y.data() + (static_cast<size_t>(ts.first) * slots + ts.second) * d);
    }
  };
  const int nt = std::max(1, std::min<int>(n_threads, static_cast<int>(jobs.size())));
  std::vector<std::thread> pool;
  for (int i = 1; i < nt; ++i) pool.emplace_back(worker);
  worker();
  for (auto& th : pool) th.join();
  if (failed) return -1;
  // 3. combine: sum_j gate_j * y_j + sum_s y_shared (+ residual)
  for (int t = 0; t < T; ++t) {
    for (int n = 0; n < d; ++n) {
      double acc = 0.0;
      for (int j = 0; j < k; ++j)
        acc += gates[static_cast<size_t>(t) * k + j] * y[(static_cast<size_t>(t) * slots + j) * d + n];
      for (int s = 0; s < S; ++s) acc += y[(static_cast<size_t>(t) * slots + k + s) * d + n];
      if (residual) acc += bf16_bits_to_double(residual[static_cast<size_t>(t) * d + n]);
      out[static_cast<size_t>(t) * d + n] = acc;
    }
  }
  if (ids_out) std::memcpy(ids_out, ids.data(), ids.size() * sizeof(int32_t));
  if (gates_out) std::memcpy(gates_out, gates.data(), gates.size() * sizeof(double));
  if (gap_out) std::memcpy(gap_out, gap.data(), gap.size() * sizeof(double));
  if (logits_out) std::memcpy(logits_out, logits.data(), logits.size() * sizeof(double));
  return 0;
}

// Grouping by expert, written from its definition: scan the experts in
// ascending id order and, for each one some token selected, list its
// selections token by token; the shared experts follow with every token.
int32_t oracle_group(const int32_t* ids, int32_t T, int32_t k, int32_t E, int32_t S, int32_t* act,
                     int32_t* off, int32_t* pair, int32_t* n_routed) {
  if (T < 0 || T > 65536 || k < 1 || E < 1 || S < 0) return -1;  // token << 8 stays within int32
  for (int i = 0; i < T * k; ++i)
    if (ids[i] < 0 || ids[i] >= E) return -1;
  int n = 0, p = 0;
  for (int e = 0; e < E; ++e) {
    const int first = p;
    for (int t = 0; t < T; ++t)
      for (int j = 0; j < k; ++j)
        if (ids[t * k + j] == e) pair[p++] = (t << 8) | j;
    if (p > first) {
      act[n] = e;
      off[n] = first;
      ++n;
    }
  }
  *n_routed = n;
  for (int s = 0; s < S; ++s) {
    act[n] = E + s;
    off[n] = p;
    ++n;
    for (int t = 0; t < T; ++t) pair[p++] = (t << 8) | (k + s);
  }
  off[n] = p;
  return n;
}

// Expert-parallel dispatch plan, from its definition: rank r of R holds the
// routed experts [r E/R, (r+1) E/R) (local id e mod E/R) and the shared
// experts (local ids E/R ..); pair i = t (k + S) + j goes to the rank holding
// expert ids[t][j] (j < k) or, for a shared slot, to the token's own rank.
// Send order: destination ranks in ascending order, each rank's pairs in
// ascending pair index. An id outside [0, E) drops its pair (position -1).
// Returns the number of dropped pairs, or -1 for bad sizes.
int32_t oracle_ep_plan(const int32_t* ids, const float* gates, int32_t T, int32_t k, int32_t S, int32_t E,
                       int32_t R, int32_t rank, int32_t* send_ids, float* send_gates, int32_t* send_token,
                       int32_t* counts, int32_t* pair_pos) {
  if (T < 0 || k < 1 || S < 0 || E < 1 || R < 1 || E % R != 0 || rank < 0 || rank >= R) return -1;
  const int slots = k + S, el = E / R, P = T * slots;
  int dropped = 0;
  for (int i = 0; i < P; ++i) {
    const int t = i / slots, j = i % slots;
    if (j < k && (ids[t * k + j] < 0 || ids[t * k + j] >= E)) {
      pair_pos[i] = -1;
      ++dropped;
    }
  }
  int pos = 0;
  for (int r = 0; r < R; ++r) {
    counts[r] = 0;
    for (int i = 0; i < P; ++i) {
      const int t = i / slots, j = i % slots;
      int dest, lid;
      float g;
      if (j < k) {
        const int e = ids[t * k + j];
        if (e < 0 || e >= E) continue;
        dest = e / el;
        lid = e % el;
        g = gates[t * k + j];
      } else {
        dest = rank;
        lid = el + (j - k);
        g = 1.0f;
      }
      if (dest != r) continue;
      pair_pos[i] = pos;
      send_ids[pos] = lid;
      send_gates[pos] = g;
      send_token[pos] = t;
      ++pos;
      ++counts[r];
    }
  }
  return dropped;
}

// Dense NVFP4 matrix times bf16 vectors: each selected row decoded
// element by element (as oracle_decode_matrix does) and dotted with x in fp64.
int oracle_dense_gemv(const oracle_matrix* m, const uint16_t* x, int32_t T, const int32_t* rows,
                      int32_t n_rows, double* out) {
  if (!m || !x || !out || m->kind != 0 || !m->codes || !m->scales || m->cols % 16 != 0 || T < 0 || n_rows < 0)
    return -1;
  const int cols = m->cols;
  const double s_t = static_cast<double>(m->tensor_scale);
  std::vector<double> w(cols), xd(static_cast<size_t>(T) * cols);
  for (size_t i = 0; i < xd.size(); ++i) xd[i] = bf16_bits_to_double(x[i]);
  for (int i = 0; i < n_rows; ++i) {
    const int r = rows ? rows[i] : i;
    if (r < 0 || r >= m->rows) return -1;
    for (int c = 0; c < cols; ++c) {
      const uint8_t byte = m->codes[static_cast<size_t>(r) * (cols / 2) + c / 2];
      const uint8_t q = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);
      const uint8_t sb = m->scales[static_cast<size_t>(r) * (cols / 16) + c / 16];
      w[c] = oracle_e2m1_decode(q) * oracle_e4m3_decode(sb) * s_t;
    }
    for (int t = 0; t < T; ++t) {
      double acc = 0.0;
      for (int c = 0; c < cols; ++c) acc += w[c] * xd[static_cast<size_t>(t) * cols + c];
      out[static_cast<size_t>(t) * n_rows + i] = acc;
    }
  }
  return 0;
}

// Attention prologue of one layer, written from its definition (fp64): per
// token and head of the fused projection qkv [T][Hq + 2*Hkv][Dh] (query heads,
// then key heads, then value heads), query and key heads are RMS-normalised
// over the head dimension and scaled by their weight vector,
//   y_i = x_i / sqrt(mean_j x_j^2 + eps) * w_i,
// then, when rope != 0, each pair (i, i + Dh/2), i < Dh/2, is rotated by the
// token's position row of the cos/sin table cs [max_pos][Dh] (cos_i in column
// i, sin_i in column Dh/2 + i):
//   out_i = y_i cos_i - y_{i+Dh/2} sin_i,   out_{i+Dh/2} = y_{i+Dh/2} cos_i + y_i sin_i;
// value heads pass unchanged. Outputs fp64: q [T][Hq][Dh], k and v
// [T][Hkv][Dh] (the values a kernel rounds to bf16 and writes to its cache
// slots). Returns 0, or -1 on a bad argument or a position outside the table.
int oracle_qk_norm_rope_kv(int32_t T, int32_t Hq, int32_t Hkv, int32_t Dh, const uint16_t* qkv, const uint16_t* q_w,
                           const uint16_t* k_w, const float* cs, int32_t max_pos, const int32_t* positions,
                           int32_t rope, double eps, double* q_out, double* k_out, double* v_out) {
  if (T < 0 || Hq < 1 || Hkv < 1 || Dh < 2 || Dh % 2 != 0 || !qkv || !q_w || !k_w || !q_out || !k_out || !v_out)
    return -1;
  if (rope && (!cs || !positions || max_pos < 1)) return -1;
  const int H = Hq + 2 * Hkv, half = Dh / 2;
  std::vector<double> x(Dh), y(Dh);
  for (int t = 0; t < T; ++t) {
    if (rope && (positions[t] < 0 || positions[t] >= max_pos)) return -1;
    for (int h = 0; h < H; ++h) {
      const uint16_t* src = qkv + (static_cast<size_t>(t) * H + h) * Dh;
      for (int i = 0; i < Dh; ++i) x[i] = bf16_bits_to_double(src[i]);
      if (h >= Hq + Hkv) {  // value head
        double* dst = v_out + (static_cast<size_t>(t) * Hkv + (h - Hq - Hkv)) * Dh;
        for (int i = 0; i < Dh; ++i) dst[i] = x[i];
        continue;
      }
      const uint16_t* w = h < Hq ? q_w : k_w;
      double ms = 0.0;
      for (int i = 0; i < Dh; ++i) ms += x[i] * x[i];
      ms /= Dh;
      const double r = 1.0 / std::sqrt(ms + eps);
      for (int i = 0; i < Dh; ++i) y[i] = x[i] * r * bf16_bits_to_double(w[i]);
      double* dst = h < Hq ? q_out + (static_cast<size_t>(t) * Hq + h) * Dh
                           : k_out + (static_cast<size_t>(t) * Hkv + (h - Hq)) * Dh;
      if (!rope) {
        for (int i = 0; i < Dh; ++i) dst[i] = y[i];
        continue;
      }
      const float* row = cs + static_cast<size_t>(positions[t]) * Dh;
      for (int i = 0; i < half; ++i) {
        const double c = row[i], s = row[half + i];
        dst[i] = y[i] * c - y[half + i] * s;
        dst[half + i] = y[half + i] * c + y[i] * s;
      }
    }
  }
  return 0;
}

// Decode attention of one layer, from its definition (fp64): query token t,
// head h attends to the cache rows start[t] .. start[t] + len[t] - 1 of key
// and value head g = h / (Hq / Hkv) (grouped-query attention):
//   s_j = (q_h . k_{g,j}) * scale,  p_j = exp(s_j - max s) / sum_j exp(s_j - max s),
//   o_h = sum_j p_j v_{g,j}.
// q bf16 [T][Hq][Dh]; k, v bf16 [rows][Hkv][Dh]; out fp64 [T][Hq][Dh]; a token
// with len 0 gets zeros. Returns 0, or -1 on a bad argument or a range outside
// [0, rows).
int oracle_decode_attention(int32_t T, int32_t Hq, int32_t Hkv, int32_t Dh, const uint16_t* q, const uint16_t* k,
                            const uint16_t* v, int64_t rows, const int64_t* start, const int32_t* len, double scale,
                            double* out) {
  if (T < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || Dh < 1 || !q || !k || !v || !start || !len || !out) return -1;
  const int group = Hq / Hkv;
  std::vector<double> sc;
  for (int t = 0; t < T; ++t) {
    if (len[t] < 0 || start[t] < 0 || start[t] + len[t] > rows) return -1;
    for (int h = 0; h < Hq; ++h) {
      const int g = h / group;
      const uint16_t* qh = q + (static_cast<size_t>(t) * Hq + h) * Dh;
      double* oh = out + (static_cast<size_t>(t) * Hq + h) * Dh;
      for (int i = 0; i < Dh; ++i) oh[i] = 0.0;
      if (len[t] == 0) continue;
      sc.assign(len[t], 0.0);
      double mx = -INFINITY;
      for (int j = 0; j < len[t]; ++j) {
        const uint16_t* kj = k + (static_cast<size_t>(start[t] + j) * Hkv + g) * Dh;
        double dot = 0.0;
        for (int i = 0; i < Dh; ++i) dot += bf16_bits_to_double(qh[i]) * bf16_bits_to_double(kj[i]);
        sc[j] = dot * scale;
        mx = std::max(mx, sc[j]);
      }
      double sum = 0.0;
      for (int j = 0; j < len[t]; ++j) {
        sc[j] = std::exp(sc[j] - mx);
        sum += sc[j];
      }
      for (int j = 0; j < len[t]; ++j) {
        const uint16_t* vj = v + (static_cast<size_t>(start[t] + j) * Hkv + g) * Dh;
        const double pj = sc[j] / sum;
        for (int i = 0; i < Dh; ++i) oh[i] += pj * bf16_bits_to_double(vj[i]);
      }
    }
  }
  return 0;
}

}  // extern "C"
