// Beam sparse-MoE layer: plain CPU oracle.
//
// TEST INFRASTRUCTURE, not part of the product.  Only the tests, the smoke
// check and the benchmark's CPU-baseline leg may load this library.  It shares
// no code, header, table or helper with the CUDA path.
//
// What it computes, and where each step comes from:
//   * router logits in FP32 from FP32 router weights; sigmoid scores; a
//     learned per-expert bias added for selection only; the best topk_group of
//     n_group expert groups; top_k experts inside them; weights normalised to
//     sum 1 and scaled by routed_scaling_factor  -- Transformers "Beam" model
//     doc, Overview ("Sparse MoE" bullet and the FP32-numerics paragraph) and
//     BeamConfig (n_group, topk_group, norm_topk_prob, routed_scaling_factor).
//   * group score = sum of the top-2 biased scores of the group -- archdb
//     "Beam-1.0-501B-A23B" fact sheet, expert-groups entry.
//   * contiguous groups of E/n_group experts ("8 groups of 32") and SwiGLU
//     experts with intermediate size 2560, no shared expert -- news article
//     "Reflection lança o Beam", section "Onde o Beam economiza ...".
//   * SwiGLU activation in FP32, RMSNorm scaling in FP32 -- "Beam" model doc,
//     Overview, FP32-numerics paragraph.
//   * sandwich RMSNorm (eps 1e-6) and the depth-scaled residual
//     r*sqrt((k-1)/k) + f/sqrt(k) -- "Beam" model doc, Overview ("Sandwich
//     norms" bullet); archdb fact sheet, residual-design entry.
//
// Numerics: every dot product accumulates in double and is rounded once to
// FP32 (the exactly rounded FP32 result up to one rounding); transcendental
// functions run in double and are rounded once.  Ties in selection go to the
// lower group / expert index.  Selected experts are reported in ascending id
// order with their weights permuted alongside; the combine sums in that order.
//
// FP8 expert weights (a reading; the pages name FP8 and NVFP4 checkpoints but no scale
// format -- news article "Reflection lança o Beam", section "Onde o Beam economiza ...";
// review page "обзор модели «Бим»", weights and vLLM-recipe entries): E4M3 codes (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no infinities,
// largest finite 448), one FP32 scale per matrix row (per output channel of a weight, per
// token row of an activation): s = fl32(amax / 448), q = e4m3(fl32(x / s)) rounded to
// nearest even and saturated to +-448.  The SwiGLU expert then runs as above with every
// GEMM input quantised that way; products of codes are exact and summed in double, and the
// two row scales are applied before the single rounding to FP32.
//
// NVFP4 expert weights (a reading, from the same passages): E2M1 codes (1 sign, 2 exponent
// bits with bias 1, 1 mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6, no infinities),
// two scales per value: one E4M3 scale per block of 16 consecutive elements of a row and one
// FP32 scale per row.  With amax the row's largest magnitude and m_b the block's:
//   s = fl32(amax / 2688)                       (2688 = 6 * 448, the two formats' maxima)
//   bs_b = e4m3( fl32( fl32(m_b / s) / 6 ) )    (nearest even, saturating)
//   q_j = e2m1( fl32( x_j / fl32(s * value(bs_b)) ) )   (nearest even, saturating to +-6)
// and a block whose scale is zero (or a row with s = 0) gets zero codes.  The value of an
// element is value(q_j) * value(bs_b) * s; a linear layer sums the exact products of codes and
// block scales in double and applies the two row scales before the single rounding to FP32.
//
// Plain loops, no BLAS, no intrinsics; std::thread over tokens.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

float bf16_bits_to_float(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return f;
}

// Round-to-nearest-even of an FP32 value to BF16 (keep the top 16 bits).
uint16_t float_to_bf16_bits(float f) {
  uint32_t u;
  std::memcpy(&u, &f, sizeof u);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u)
    return static_cast<uint16_t>((u >> 16) | 0x0040u);  // quiet NaN
  const uint32_t lower = u & 0xffffu;
  uint32_t upper = u >> 16;
  if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
  return static_cast<uint16_t>(upper);
}

int resolve_threads(int nthreads) {
  if (nthreads > 0) return nthreads;
  unsigned hc = std::thread::hardware_concurrency();
  return hc ? static_cast<int>(hc) : 1;
}

template <class F>
void parallel_for(int64_t n, int nthreads, F body) {
  nthreads = resolve_threads(nthreads);
  if (nthreads <= 1 || n <= 1) {
    for (int64_t i = 0; i < n; ++i) body(i);
    return;
  }
  if (nthreads > n) nthreads = static_cast<int>(n);
  std::vector<std::thread> pool;
  pool.reserve(nthreads);
  for (int w = 0; w < nthreads; ++w) {
    pool.emplace_back([=, &body] {
      for (int64_t i = w; i < n; i += nthreads) body(i);
    });
  }
  for (auto& th : pool) th.join();
}

double sigmoid(double x) { return 1.0 / (1.0 + std::exp(-x)); }

// E4M3 code -> value.  Exponent field 0 holds the subnormals m/8 * 2^-6; S.1111.111 is NaN.
double e4m3_value(uint8_t b) {
  const int sgn = b >> 7, e = (b >> 3) & 15, m = b & 7;
  if (e == 15 && m == 7) return std::nan("");
  const double v = e == 0 ? std::ldexp(m / 8.0, -6) : std::ldexp(1.0 + m / 8.0, e - 7);
  return sgn ? -v : v;
}

// Value -> E4M3 code, round to nearest with ties to the even code, saturating to +-448.
uint8_t e4m3_code(float f) {
  if (std::isnan(f)) return 0x7f;
  const uint8_t sgn = std::signbit(f) ? 0x80 : 0x00;
  const double a = std::fabs(static_cast<double>(f));
  uint8_t mag;
  if (a >= 448.0) {
    mag = 0x7e;
  } else if (a < std::ldexp(1.0, -6)) {
    // subnormal range: steps of 2^-9; rounding up to 8 steps gives the smallest normal (code 8)
    mag = static_cast<uint8_t>(std::nearbyint(a / std::ldexp(1.0, -9)));
  } else {
    int ex;
    std::frexp(a, &ex);  // a = f * 2^ex, f in [0.5, 1): a in [2^(ex-1), 2^ex)
    const int E = ex - 1;
    double r = std::nearbyint(a / std::ldexp(1.0, E - 3));  // 8 .. 16 steps of 2^(E-3)
    int Eb = E + 7;
    if (r == 16.0) {
      r = 8.0;
      ++Eb;
    }
    const int code = (Eb << 3) | (static_cast<int>(r) - 8);
    mag = static_cast<uint8_t>(code > 0x7e ? 0x7e : code);
  }
  return static_cast<uint8_t>(sgn | mag);
}

// Quantises one BF16 row of n values: s = fl32(amax / 448), q_j = e4m3(fl32(x_j / s)).
// An all-zero row gets s = 0 and zero codes.
float quantize_row(int64_t n, const uint16_t* x, uint8_t* q) {
  float amax = 0.0f;
  for (int64_t j = 0; j < n; ++j) amax = std::max(amax, std::fabs(bf16_bits_to_float(x[j])));
  const float s = amax / 448.0f;
  for (int64_t j = 0; j < n; ++j)
    q[j] = s > 0.0f ? e4m3_code(bf16_bits_to_float(x[j]) / s) : 0;
  return s;
}

// y_c = fl32( sx * sw_c * sum_j value(xq_j) * value(Wq[c, j]) ) for c < n_out; Wq is [n_out, K].
void linear_fp8_row(int64_t K, int64_t n_out, const uint8_t* xq, float sx, const uint8_t* Wq,
                    const float* sw, float* y) {
  double value[256];  // e4m3_value of every code, looked up below
  for (int b = 0; b < 256; ++b) value[b] = e4m3_value(static_cast<uint8_t>(b));
  std::vector<double> xv(K);
  for (int64_t j = 0; j < K; ++j) xv[j] = value[xq[j]];
  for (int64_t c = 0; c < n_out; ++c) {
    const uint8_t* w = Wq + c * K;
    double acc = 0.0;
    for (int64_t j = 0; j < K; ++j) acc += xv[j] * value[w[j]];
    y[c] = static_cast<float>(static_cast<double>(sx) * static_cast<double>(sw[c]) * acc);
  }
}

// E2M1 code -> value.  Bit 3 is the sign; exponent field e = bits 2..1, mantissa bit 0:
// e = 0 gives m * 0.5 (0 or 0.5), e > 0 gives 2^(e-1) * (1 + m/2).
double e2m1_value(uint8_t c) {
  const int e = (c >> 1) & 3, m = c & 1;
  const double v = e == 0 ? 0.5 * m : std::ldexp(1.0 + 0.5 * m, e - 1);
  return (c & 8) ? -v : v;
}

// Value -> E2M1 code, round to nearest with ties to the even code, saturating to +-6.  Inside
// each binade the grid step is constant (0.5 below 2, 1 on [2, 4), 2 on [4, 6]), so the value
// is rounded to a whole number of steps; an even step count is an even code.
uint8_t e2m1_code(float f) {
  const uint8_t sgn = std::signbit(f) ? 8 : 0;
  const double a = std::fabs(static_cast<double>(f));
  uint8_t mag;
  if (a >= 6.0) {
    mag = 7;
  } else if (a < 2.0) {
    mag = static_cast<uint8_t>(std::nearbyint(a / 0.5));  // 0..4 halves: codes 0..4
  } else if (a < 4.0) {
    mag = static_cast<uint8_t>(std::nearbyint(a) + 2.0);  // 2..4: codes 4..6
  } else {
    mag = static_cast<uint8_t>(std::nearbyint(a / 2.0) + 4.0);  // 2..3 (x2): codes 6..7
  }
  return static_cast<uint8_t>(sgn | mag);
}

// NVFP4 quantisation of one BF16 row of n values (n a multiple of 16): q [n] codes (one per
// byte), bs [n / 16] E4M3 block-scale codes; returns the row scale s.
float quantize_row_nvfp4(int64_t n, const uint16_t* x, uint8_t* q, uint8_t* bs) {
  float amax = 0.0f;
  for (int64_t j = 0; j < n; ++j) amax = std::max(amax, std::fabs(bf16_bits_to_float(x[j])));
  const float s = amax / 2688.0f;
  for (int64_t b = 0; b < n / 16; ++b) {
    const uint16_t* xb = x + b * 16;
    float mb = 0.0f;
    for (int j = 0; j < 16; ++j) mb = std::max(mb, std::fabs(bf16_bits_to_float(xb[j])));
    float t = 0.0f;
    if (s > 0.0f) {
      t = mb / s;
      t = t / 6.0f;
    }
    bs[b] = s > 0.0f ? e4m3_code(t) : 0;
    const float den = s * static_cast<float>(e4m3_value(bs[b]));
    for (int j = 0; j < 16; ++j)
      q[b * 16 + j] = den > 0.0f ? e2m1_code(bf16_bits_to_float(xb[j]) / den) : 0;
  }
  return s;
}

// y_c = fl32( sx * sw_c * sum_b value(xbs_b) value(Wbs[c, b]) sum_{j in b} value(xq_j)
// value(Wq[c, j]) ) for c < n_out; Wq [n_out, K] codes, Wbs [n_out, K / 16] block scales.
void linear_nvfp4_row(int64_t K, int64_t n_out, const uint8_t* xq, const uint8_t* xbs, float sx,
                      const uint8_t* Wq, const uint8_t* Wbs, const float* sw, float* y) {
  double v4[16];
  for (int c = 0; c < 16; ++c) v4[c] = e2m1_value(static_cast<uint8_t>(c));
  const int64_t nb = K / 16;
  for (int64_t c = 0; c < n_out; ++c) {
    const uint8_t* w = Wq + c * K;
    const uint8_t* wb = Wbs + c * nb;
    double acc = 0.0;
    for (int64_t b = 0; b < nb; ++b) {
      double part = 0.0;
      for (int j = 0; j < 16; ++j) part += v4[xq[b * 16 + j] & 15] * v4[w[b * 16 + j] & 15];
      acc += e4m3_value(xbs[b]) * e4m3_value(wb[b]) * part;
    }
    y[c] = static_cast<float>(static_cast<double>(sx) * static_cast<double>(sw[c]) * acc);
  }
}

// out[n, c] = fl32( sum_j w[t, j] * ys[n, j, c] ) over the k slots in their order, t = tokens[n].
void combine_slots(int64_t ntok, const int64_t* tokens, int64_t d, int k, const float* w,
                   const float* ys, float* out) {
  for (int64_t n = 0; n < ntok; ++n) {
    const int64_t t = tokens[n];
    for (int64_t c = 0; c < d; ++c) {
      double acc = 0.0;
      for (int j = 0; j < k; ++j)
        acc += static_cast<double>(w[t * k + j]) *
               static_cast<double>(ys[(static_cast<size_t>(n) * k + j) * d + c]);
      out[n * d + c] = static_cast<float>(acc);
    }
  }
}

}  // namespace

extern "C" {

int oracle_hardware_threads(void) { return resolve_threads(0); }

void oracle_f32_to_bf16(int64_t n, const float* in, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = float_to_bf16_bits(in[i]);
}

void oracle_bf16_to_f32(int64_t n, const uint16_t* in, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = bf16_bits_to_float(in[i]);
}

// logits[t, e] = fl32( sum_j h[t, j] * Wr[e, j] ), h BF16 widened exactly.
void oracle_router_logits(int64_t T, int64_t d, int64_t E, const uint16_t* h,
                          const float* Wr, float* logits, int nthreads) {
  parallel_for(T, nthreads, [&](int64_t t) {
    const uint16_t* ht = h + t * d;
    for (int64_t e = 0; e < E; ++e) {
      const float* we = Wr + e * d;
      double acc = 0.0;
      for (int64_t j = 0; j < d; ++j)
        acc += static_cast<double>(bf16_bits_to_float(ht[j])) * static_cast<double>(we[j]);
      logits[t * E + e] = static_cast<float>(acc);
    }
  });
}

// Selection and weights for T tokens from their router logits.
//   s  = sigmoid(logit)                  (FP32)
//   sb = s + bias                        (FP32; used only to choose)
//   group score gs_g = sum of the top-2 sb in group g (top-1 if a group has one expert)
//   keep the topk_group groups with the largest gs (lower g wins ties)
//   choose the top_k experts with the largest sb among kept groups (lower e wins ties)
//   w = S * s / sum(s over the chosen)   (or S * s without normalisation)
// idx[t, :] lists the chosen experts in ascending id; w[t, :] follows it.
// margin_expert[t] = sb of the k-th chosen minus sb of the best unchosen expert in a
// kept group (+inf if none); margin_group[t] = gs of the last kept group minus gs of
// the best dropped group (+inf if none).  Either margin array may be NULL.
// Returns 0, or -1 on an invalid shape.
int oracle_route(int64_t T, int E, int G, int Gk, int k, float S, int norm_topk_prob,
                 const float* logits, const float* bias, int32_t* idx, float* w,
                 float* margin_expert, float* margin_group, int nthreads) {
  if (E <= 0 || G <= 0 || E % G != 0 || Gk <= 0 || Gk > G || k <= 0 ||
      k > Gk * (E / G))
    return -1;
  const int per = E / G;
  parallel_for(T, nthreads, [&](int64_t t) {
    const float* lt = logits + t * E;
    std::vector<float> s(E), sb(E);
    for (int e = 0; e < E; ++e) {
      s[e] = static_cast<float>(sigmoid(static_cast<double>(lt[e])));
      sb[e] = s[e] + bias[e];
    }
    // group scores
    std::vector<float> gs(G);
    for (int g = 0; g < G; ++g) {
      std::vector<float> v(sb.begin() + g * per, sb.begin() + (g + 1) * per);
      std::sort(v.begin(), v.end(), [](float a, float b) { return a > b; });
      gs[g] = per >= 2 ? v[0] + v[1] : v[0];
    }
    std::vector<int> gorder(G);
    for (int g = 0; g < G; ++g) gorder[g] = g;
    std::sort(gorder.begin(), gorder.end(), [&](int a, int b) {
      if (gs[a] != gs[b]) return gs[a] > gs[b];
      return a < b;
    });
    std::vector<char> kept(G, 0);
    for (int i = 0; i < Gk; ++i) kept[gorder[i]] = 1;
    // candidate experts in kept groups, best first
    std::vector<int> cand;
    for (int e = 0; e < E; ++e)
      if (kept[e / per]) cand.push_back(e);
    std::sort(cand.begin(), cand.end(), [&](int a, int b) {
      if (sb[a] != sb[b]) return sb[a] > sb[b];
      return a < b;
    });
    std::vector<int> chosen(cand.begin(), cand.begin() + k);
    std::sort(chosen.begin(), chosen.end());
    double denom = 0.0;
    for (int e : chosen) denom += static_cast<double>(s[e]);
    for (int j = 0; j < k; ++j) {
      const int e = chosen[j];
      idx[t * k + j] = e;
      const double num = static_cast<double>(S) * static_cast<double>(s[e]);
      w[t * k + j] = static_cast<float>(norm_topk_prob ? num / denom : num);
    }
    const float inf = std::numeric_limits<float>::infinity();
    if (margin_expert)
      margin_expert[t] = static_cast<int>(cand.size()) > k ? sb[cand[k - 1]] - sb[cand[k]] : inf;
    if (margin_group)
      margin_group[t] = G > Gk ? gs[gorder[Gk - 1]] - gs[gorder[Gk]] : inf;
  });
  return 0;
}

// One SwiGLU expert on one input row x [d] (BF16):
//   g_i = fl32(sum_j x_j Wg[i, j]),  u_i = fl32(sum_j x_j Wu[i, j])
//   a_i = bf16( fl32(silu(g_i)) * u_i ),  silu(g) = g / (1 + exp(-g))
//   y_c = fl32(sum_i a_i Wd[c, i])
// Wg, Wu are [I, d]; Wd is [d, I] (nn.Linear out x in).  a_out [I] (BF16 bits) may be NULL.
void oracle_expert_mlp(int64_t d, int64_t I, const uint16_t* x, const uint16_t* Wg,
                       const uint16_t* Wu, const uint16_t* Wd, float* y, uint16_t* a_out) {
  std::vector<double> xd(d);
  for (int64_t j = 0; j < d; ++j) xd[j] = bf16_bits_to_float(x[j]);
  std::vector<double> a(I);
  for (int64_t i = 0; i < I; ++i) {
    double gacc = 0.0, uacc = 0.0;
    const uint16_t* wg = Wg + i * d;
    const uint16_t* wu = Wu + i * d;
    for (int64_t j = 0; j < d; ++j) {
      gacc += xd[j] * static_cast<double>(bf16_bits_to_float(wg[j]));
      uacc += xd[j] * static_cast<double>(bf16_bits_to_float(wu[j]));
    }
    const float g = static_cast<float>(gacc);
    const float u = static_cast<float>(uacc);
    const float act = static_cast<float>(static_cast<double>(g) * sigmoid(static_cast<double>(g)));
    const uint16_t ab = float_to_bf16_bits(act * u);
    if (a_out) a_out[i] = ab;
    a[i] = bf16_bits_to_float(ab);
  }
  for (int64_t c = 0; c < d; ++c) {
    const uint16_t* wd = Wd + c * I;
    double acc = 0.0;
    for (int64_t i = 0; i < I; ++i) acc += a[i] * static_cast<double>(bf16_bits_to_float(wd[i]));
    y[c] = static_cast<float>(acc);
  }
}

// MoE output for a list of tokens: out[n, c] = fl32( sum_j w[t, j] * y_{idx[t, j]}[c] )
// summed in the order of idx (ascending expert id), t = tokens[n].  Expert weights
// are passed as per-expert pointer arrays so that callers may supply only the
// experts these tokens use; a NULL entry that is needed makes the call return -1.
int oracle_moe_tokens(int64_t ntok, const int64_t* tokens, int64_t d, int64_t I, int k,
                      const uint16_t* h, const int32_t* idx, const float* w,
                      const uint16_t* const* Wg, const uint16_t* const* Wu,
                      const uint16_t* const* Wd, float* out, int nthreads) {
  for (int64_t n = 0; n < ntok; ++n)
    for (int j = 0; j < k; ++j) {
      const int e = idx[tokens[n] * k + j];
      if (!Wg[e] || !Wu[e] || !Wd[e]) return -1;
    }
  // one work item per (token, slot); the reduction over slots runs afterwards in order
  std::vector<float> ys(static_cast<size_t>(ntok) * k * d);
  parallel_for(ntok * k, nthreads, [&](int64_t item) {
    const int64_t n = item / k;
    const int j = static_cast<int>(item % k);
    const int64_t t = tokens[n];
    const int e = idx[t * k + j];
    oracle_expert_mlp(d, I, h + t * d, Wg[e], Wu[e], Wd[e], ys.data() + item * d, nullptr);
  });
  combine_slots(ntok, tokens, d, k, w, ys.data(), out);
  return 0;
}

void oracle_f32_to_e4m3(int64_t n, const float* in, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_code(in[i]);
}

void oracle_e4m3_to_f32(int64_t n, const uint8_t* in, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = static_cast<float>(e4m3_value(in[i]));
}

// Row-wise E4M3 quantisation of a BF16 matrix [rows, cols] (see quantize_row).
void oracle_quantize_rows_e4m3(int64_t rows, int64_t cols, const uint16_t* x, uint8_t* q,
                               float* scale, int nthreads) {
  parallel_for(rows, nthreads,
               [&](int64_t r) { scale[r] = quantize_row(cols, x + r * cols, q + r * cols); });
}

// FP8 linear layer on quantised rows: y[r, c] = fl32( sx_r * sw_c * sum_j xq[r, j] Wq[c, j] )
// with codes decoded exactly; xq [rows, K], Wq [n_out, K].
void oracle_linear_fp8(int64_t rows, int64_t n_out, int64_t K, const uint8_t* xq,
                       const float* sx, const uint8_t* Wq, const float* sw, float* y,
                       int nthreads) {
  parallel_for(rows, nthreads, [&](int64_t r) {
    linear_fp8_row(K, n_out, xq + r * K, sx[r], Wq, sw, y + r * n_out);
  });
}

// One SwiGLU expert with E4M3 weights on one input row x [d] (BF16):
//   (xq, sx) = quantize(x)
//   g = linear_fp8(xq, sx; Wgq, sg),  u = linear_fp8(xq, sx; Wuq, su)      [I]
//   a_i = bf16( fl32(silu(g_i)) * u_i )
//   (aq, sa) = quantize(a)
//   y = linear_fp8(aq, sa; Wdq, sd)                                          [d]
// Wgq, Wuq [I, d] with row scales sg, su [I]; Wdq [d, I] with row scales sd [d].
// a_out [I] (BF16 bits, before its quantisation) may be NULL.
void oracle_expert_mlp_fp8(int64_t d, int64_t I, const uint16_t* x, const uint8_t* Wgq,
                           const float* sg, const uint8_t* Wuq, const float* su,
                           const uint8_t* Wdq, const float* sd, float* y, uint16_t* a_out) {
  std::vector<uint8_t> xq(d), aq(I);
  const float sx = quantize_row(d, x, xq.data());
  std::vector<float> g(I), u(I);
  linear_fp8_row(d, I, xq.data(), sx, Wgq, sg, g.data());
  linear_fp8_row(d, I, xq.data(), sx, Wuq, su, u.data());
  std::vector<uint16_t> a(I);
  for (int64_t i = 0; i < I; ++i) {
    const float act =
        static_cast<float>(static_cast<double>(g[i]) * sigmoid(static_cast<double>(g[i])));
    a[i] = float_to_bf16_bits(act * u[i]);
  }
  if (a_out) std::copy(a.begin(), a.end(), a_out);
  const float sa = quantize_row(I, a.data(), aq.data());
  linear_fp8_row(I, d, aq.data(), sa, Wdq, sd, y);
}

// MoE output for a list of tokens with E4M3 experts; as oracle_moe_tokens otherwise.
int oracle_moe_tokens_fp8(int64_t ntok, const int64_t* tokens, int64_t d, int64_t I, int k,
                          const uint16_t* h, const int32_t* idx, const float* w,
                          const uint8_t* const* Wgq, const float* const* sg,
                          const uint8_t* const* Wuq, const float* const* su,
                          const uint8_t* const* Wdq, const float* const* sd, float* out,
                          int nthreads) {
  for (int64_t n = 0; n < ntok; ++n)
    for (int j = 0; j < k; ++j) {
      const int e = idx[tokens[n] * k + j];
      if (!Wgq[e] || !sg[e] || !Wuq[e] || !su[e] || !Wdq[e] || !sd[e]) return -1;
    }
  std::vector<float> ys(static_cast<size_t>(ntok) * k * d);
  parallel_for(ntok * k, nthreads, [&](int64_t item) {
    const int64_t n = item / k;
    const int j = static_cast<int>(item % k);
    const int64_t t = tokens[n];
    const int e = idx[t * k + j];
    oracle_expert_mlp_fp8(d, I, h + t * d, Wgq[e], sg[e], Wuq[e], su[e], Wdq[e], sd[e],
                          ys.data() + item * d, nullptr);
  });
  combine_slots(ntok, tokens, d, k, w, ys.data(), out);
  return 0;
}

void oracle_f32_to_e2m1(int64_t n, const float* in, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e2m1_code(in[i]);
}

void oracle_e2m1_to_f32(int64_t n, const uint8_t* in, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = static_cast<float>(e2m1_value(in[i]));
}

// Row-wise NVFP4 quantisation of a BF16 matrix [rows, cols] (see quantize_row_nvfp4):
// q [rows, cols] codes, bs [rows, cols / 16] block scales, scale [rows].
void oracle_quantize_rows_nvfp4(int64_t rows, int64_t cols, const uint16_t* x, uint8_t* q,
                                uint8_t* bs, float* scale, int nthreads) {
  parallel_for(rows, nthreads, [&](int64_t r) {
    scale[r] = quantize_row_nvfp4(cols, x + r * cols, q + r * cols, bs + r * (cols / 16));
  });
}

// NVFP4 linear layer on quantised rows (see linear_nvfp4_row): xq [rows, K], xbs [rows, K/16],
// sx [rows]; Wq [n_out, K], Wbs [n_out, K/16], sw [n_out]; y [rows, n_out].
void oracle_linear_nvfp4(int64_t rows, int64_t n_out, int64_t K, const uint8_t* xq,
                         const uint8_t* xbs, const float* sx, const uint8_t* Wq,
                         const uint8_t* Wbs, const float* sw, float* y, int nthreads) {
  parallel_for(rows, nthreads, [&](int64_t r) {
    linear_nvfp4_row(K, n_out, xq + r * K, xbs + r * (K / 16), sx[r], Wq, Wbs, sw,
                     y + r * n_out);
  });
}

// One SwiGLU expert with NVFP4 weights on one BF16 input row, as oracle_expert_mlp_fp8 with
// every quantisation in NVFP4: Wgq, Wuq [I, d] codes with block scales [I, d/16] and row
// scales [I]; Wdq [d, I] with [d, I/16] and [d].  a_out [I] (BF16 bits before the activation's
// quantisation) may be NULL.
void oracle_expert_mlp_nvfp4(int64_t d, int64_t I, const uint16_t* x, const uint8_t* Wgq,
                             const uint8_t* Wgb, const float* sg, const uint8_t* Wuq,
                             const uint8_t* Wub, const float* su, const uint8_t* Wdq,
                             const uint8_t* Wdb, const float* sd, float* y, uint16_t* a_out) {
  std::vector<uint8_t> xq(d), xb(d / 16), aq(I), ab(I / 16);
  const float sx = quantize_row_nvfp4(d, x, xq.data(), xb.data());
  std::vector<float> g(I), u(I);
  linear_nvfp4_row(d, I, xq.data(), xb.data(), sx, Wgq, Wgb, sg, g.data());
  linear_nvfp4_row(d, I, xq.data(), xb.data(), sx, Wuq, Wub, su, u.data());
  std::vector<uint16_t> a(I);
  for (int64_t i = 0; i < I; ++i) {
    const float act =
        static_cast<float>(static_cast<double>(g[i]) * sigmoid(static_cast<double>(g[i])));
    a[i] = float_to_bf16_bits(act * u[i]);
  }
  if (a_out) std::copy(a.begin(), a.end(), a_out);
  const float sa = quantize_row_nvfp4(I, a.data(), aq.data(), ab.data());
  linear_nvfp4_row(I, d, aq.data(), ab.data(), sa, Wdq, Wdb, sd, y);
}

// MoE output for a list of tokens with NVFP4 experts; as oracle_moe_tokens otherwise.
int oracle_moe_tokens_nvfp4(int64_t ntok, const int64_t* tokens, int64_t d, int64_t I, int k,
                            const uint16_t* h, const int32_t* idx, const float* w,
                            const uint8_t* const* Wgq, const uint8_t* const* Wgb,
                            const float* const* sg, const uint8_t* const* Wuq,
                            const uint8_t* const* Wub, const float* const* su,
                            const uint8_t* const* Wdq, const uint8_t* const* Wdb,
                            const float* const* sd, float* out, int nthreads) {
  for (int64_t n = 0; n < ntok; ++n)
    for (int j = 0; j < k; ++j) {
      const int e = idx[tokens[n] * k + j];
      if (!Wgq[e] || !Wgb[e] || !sg[e] || !Wuq[e] || !Wub[e] || !su[e] || !Wdq[e] || !Wdb[e] ||
          !sd[e])
        return -1;
    }
  std::vector<float> ys(static_cast<size_t>(ntok) * k * d);
  parallel_for(ntok * k, nthreads, [&](int64_t item) {
    const int64_t n = item / k;
    const int j = static_cast<int>(item % k);
    const int64_t t = tokens[n];
    const int e = idx[t * k + j];
    oracle_expert_mlp_nvfp4(d, I, h + t * d, Wgq[e], Wgb[e], sg[e], Wuq[e], Wub[e], su[e],
                            Wdq[e], Wdb[e], sd[e], ys.data() + item * d, nullptr);
  });
  combine_slots(ntok, tokens, d, k, w, ys.data(), out);
  return 0;
}

// RMSNorm in FP32 semantics: y = fl32( x / sqrt(mean(x^2) + eps) * g ), row-wise over [T, d].
void oracle_rmsnorm(int64_t T, int64_t d, const float* x, const float* g, float eps, float* y,
                    int nthreads) {
  parallel_for(T, nthreads, [&](int64_t t) {
    const float* xt = x + t * d;
    double ss = 0.0;
    for (int64_t j = 0; j < d; ++j) ss += static_cast<double>(xt[j]) * static_cast<double>(xt[j]);
    const double rms = std::sqrt(ss / static_cast<double>(d) + static_cast<double>(eps));
    for (int64_t j = 0; j < d; ++j)
      y[t * d + j] = static_cast<float>(static_cast<double>(xt[j]) / rms * static_cast<double>(g[j]));
  });
}

// Depth-scaled residual after the k-th contribution:
//   out = fl32( x * sqrt((k-1)/k) + f * (1/sqrt(k)) ).
void oracle_residual(int64_t n, const float* x, const float* f, int k, float* out) {
  const double kk = static_cast<double>(k);
  const double cx = std::sqrt((kk - 1.0) / kk);
  const double cf = 1.0 / std::sqrt(kk);
  for (int64_t i = 0; i < n; ++i)
    out[i] = static_cast<float>(static_cast<double>(x[i]) * cx + static_cast<double>(f[i]) * cf);
}

// Selection-bias update after one step (auxiliary-loss-free balancing): experts that got fewer
// than the mean number of slots gain gamma, experts that got more lose gamma:
//   bias'[e] = fl32( bias[e] + gamma * sign(slots / E - counts[e]) ),  sign(0) = 0.
void oracle_bias_update(int E, const int32_t* counts, int64_t slots, const float* bias,
                        float gamma, float* bias_out) {
  const double mean = static_cast<double>(slots) / static_cast<double>(E);
  for (int e = 0; e < E; ++e) {
    const double c = static_cast<double>(counts[e]);
    const float sgn = c < mean ? 1.0f : (c > mean ? -1.0f : 0.0f);
    bias_out[e] = bias[e] + gamma * sgn;
  }
}

void oracle_residual_coefficients(int k, double* cx, double* cf) {
  const double kk = static_cast<double>(k);
  *cx = std::sqrt((kk - 1.0) / kk);
  *cf = 1.0 / std::sqrt(kk);
}

}  // extern "C"
