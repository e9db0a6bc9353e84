// Plain CPU oracle for the forward pass of one sparse Mixture-of-Experts layer.
//
// TEST INFRASTRUCTURE ONLY. The tests, the package's smoke() and the bench's
// CPU-baseline leg call this library to check and to time the CUDA path; the
// product path never loads it. It shares no source, header, table or helper
// with the CUDA library: every step below is written out from its definition.
//
// What it computes, step by step (page titles abbreviated as
//   [P2] "Kimi K3: The Open Model That Just Cornered the AI Frontier",
//   [P3] "Kimi K3: Open Frontier Intelligence"):
//
//  1. Router logits l[t,e] = sum_i x[t,i] * W_router[i,e] (+ b[e]).
//     [P2] section "Mixture-of-Experts with Dynamic Load Balancing", gating
//     code: one linear gate projection from d_model to n_experts.
//     The pages fix no precision for it; reading taken: fp32, with x widened
//     from bf16 exactly, in a stated order (oracle_router_logits below), so
//     that routing decisions are reproducible bit for bit.
//  2. probs = softmax over ALL experts ([P2] gating code: softmax is taken
//     over the last axis before top-k). Computed here in fp64.
//  3. top-k: the k largest, returned with their (unnormalised) softmax values
//     ([P2] gating code returns the top-k values and indices as they are).
//     Selection compares the fp32 logits (softmax is monotone, so this is the
//     same set as ranking the probabilities in exact arithmetic); equal
//     logits go to the lower expert index; slots are in descending order.
//  4. dispatch: a stable counting sort of the (token, slot) pairs by expert
//     ([P3] section "Operational Execution Flow": tokens are dispatched to
//     their active routed experts).
//  5. per-expert SwiGLU FFN in fp64: g = x W_gu[:, 0:f], u = x W_gu[:, f:2f],
//     h = SiLU(g) * u with SiLU(a) = a / (1 + exp(-a)), y = h W_down.
//  6. combine: out[t] = sum_j p[t,j] * y[t,j] in fp64 ([P3] "Operational
//     Execution Flow": the routed output is the probability-weighted sum of
//     the selected experts' outputs).
//
// Build: g++ -O2 -std=c++17 -fopenmp -ffp-contract=off -mfma -shared -fPIC.
// -ffp-contract=off keeps the compiler from fusing any multiply-add the code
// does not spell as std::fma; -mfma makes std::fma a single instruction.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <functional>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

inline float bf16_to_float(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, sizeof(f));
  return f;
}

inline double bf16_to_double(uint16_t b) { return static_cast<double>(bf16_to_float(b)); }

constexpr int64_t kChunk = 128;  // router summation chunk (step 1)

}  // namespace

extern "C" {

// Status codes: 0 ok, 1 bad argument, 2 non-finite input.

int oracle_version(void) { return 1; }

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

// Step 1. logits[t*E + e] in fp32.
// Order: i runs over consecutive chunks of 128 indices. Inside chunk c the
// partial p_c starts at +0 and takes p_c = fma(x_i, W[i,e], p_c) for i
// ascending. Then l = p_0, l = l + p_1, ..., l = l + p_{C-1} (ascending c),
// then l = l + b_e when a bias is given. Every operation is one correctly
// rounded fp32 fma or add.
int oracle_router_logits(const uint16_t* x, const float* Wr, const float* bias,
                         int64_t T, int64_t d, int64_t E, float* logits) {
  if (!x || !Wr || !logits || T < 0 || d <= 0 || E <= 0) return 1;
  const int64_t C = (d + kChunk - 1) / kChunk;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
  for (int64_t t = 0; t < T; ++t) {
    std::vector<float> l(E), p(E);
    std::vector<float> xf(d);
    for (int64_t i = 0; i < d; ++i) {
      xf[i] = bf16_to_float(x[t * d + i]);
      if (!std::isfinite(xf[i])) bad |= 1;
    }
    for (int64_t c = 0; c < C; ++c) {
      std::fill(p.begin(), p.end(), 0.0f);
      const int64_t i0 = c * kChunk, i1 = std::min(d, i0 + kChunk);
      for (int64_t i = i0; i < i1; ++i) {
        const float xi = xf[i];
        const float* w = Wr + i * E;
        for (int64_t e = 0; e < E; ++e) p[e] = std::fma(xi, w[e], p[e]);
      }
      if (c == 0) {
        for (int64_t e = 0; e < E; ++e) l[e] = p[e];
      } else {
        for (int64_t e = 0; e < E; ++e) l[e] = l[e] + p[e];
      }
    }
    if (bias)
      for (int64_t e = 0; e < E; ++e) l[e] = l[e] + bias[e];
    for (int64_t e = 0; e < E; ++e) logits[t * E + e] = l[e];
  }
  return bad ? 2 : 0;
}

// Steps 2 and 3. For each token: probabilities over all E experts in fp64,
// then the k experts with the largest logits (ties: lower index first), in
// descending order, with their unnormalised probabilities.
// probs (optional, may be NULL) receives all E probabilities.
int oracle_topk(const float* logits, int64_t T, int64_t E, int64_t k,
                int32_t* idx, double* w, double* probs) {
  if (!logits || !idx || !w || T < 0 || E <= 0 || k <= 0 || k > E) return 1;
  int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
  for (int64_t t = 0; t < T; ++t) {
    const float* l = logits + t * E;
    double m = -INFINITY;
    for (int64_t e = 0; e < E; ++e) {
      if (!std::isfinite(l[e])) bad |= 1;
      m = std::max(m, static_cast<double>(l[e]));
    }
    double s = 0.0;
    for (int64_t e = 0; e < E; ++e) s += std::exp(static_cast<double>(l[e]) - m);
    std::vector<int32_t> order(E);
    for (int64_t e = 0; e < E; ++e) order[e] = static_cast<int32_t>(e);
    // stable: among equal logits the original (ascending) index order stays
    std::stable_sort(order.begin(), order.end(),
                     [l](int32_t a, int32_t b) { return l[a] > l[b]; });
    for (int64_t j = 0; j < k; ++j) {
      const int32_t e = order[j];
      idx[t * k + j] = e;
      w[t * k + j] = std::exp(static_cast<double>(l[e]) - m) / s;
    }
    if (probs)
      for (int64_t e = 0; e < E; ++e) probs[t * E + e] = std::exp(static_cast<double>(l[e]) - m) / s;
  }
  return bad ? 2 : 0;
}

// Step 4. Stable counting sort of the T*k (token, slot) pairs by expert.
// counts[e]; offsets[0..E] (exclusive scan, offsets[E] = T*k); perm_token[r]
// is the token of permuted row r; inv_perm[t*k + j] is the row of (t, j).
// Inside one expert the rows follow ascending token order.
int oracle_permute(const int32_t* idx, int64_t T, int64_t E, int64_t k,
                   int32_t* counts, int32_t* offsets, int32_t* perm_token, int32_t* inv_perm) {
  if (!idx || !counts || !offsets || !perm_token || !inv_perm || T < 0 || E <= 0 || k <= 0) return 1;
  for (int64_t e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t q = 0; q < T * k; ++q) {
    const int32_t e = idx[q];
    if (e < 0 || e >= E) return 1;
    counts[e] += 1;
  }
  offsets[0] = 0;
  for (int64_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  std::vector<int32_t> cursor(offsets, offsets + E);
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t j = 0; j < k; ++j) {
      const int32_t e = idx[t * k + j];
      const int32_t r = cursor[e]++;
      perm_token[r] = static_cast<int32_t>(t);
      inv_perm[t * k + j] = r;
    }
  }
  return 0;
}

// Step 5 for one expert: n input rows x_rows[n, d] (bf16) through that
// expert's W_gu[d, 2f] and W_down[f, d] (bf16), output y[n, d] in fp64.
// h (optional, may be NULL) receives SiLU(g)*u as [n, f] fp64.
int oracle_expert_ffn(const uint16_t* x_rows, int64_t n, const uint16_t* Wgu, const uint16_t* Wd,
                      int64_t d, int64_t f, double* y, double* h_out) {
  if ((!x_rows && n > 0) || !Wgu || !Wd || !y || n < 0 || d <= 0 || f <= 0) return 1;
  const int64_t f2 = 2 * f;
  const int64_t R = 16;  // rows per block (only to reuse a widened weight row)
  const int64_t nblk = (n + R - 1) / R;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t b = 0; b < nblk; ++b) {
    const int64_t r0 = b * R, r1 = std::min(n, r0 + R), nr = r1 - r0;
    std::vector<double> gu(nr * f2, 0.0), hrow(nr * f), yy(nr * d, 0.0), wrow(std::max(f2, d));
    for (int64_t i = 0; i < d; ++i) {
      for (int64_t j = 0; j < f2; ++j) wrow[j] = bf16_to_double(Wgu[i * f2 + j]);
      for (int64_t r = 0; r < nr; ++r) {
        const double xi = bf16_to_double(x_rows[(r0 + r) * d + i]);
        double* acc = &gu[r * f2];
        for (int64_t j = 0; j < f2; ++j) acc[j] += xi * wrow[j];
      }
    }
    for (int64_t r = 0; r < nr; ++r)
      for (int64_t j = 0; j < f; ++j) {
        const double g = gu[r * f2 + j], u = gu[r * f2 + f + j];
        const double silu = g / (1.0 + std::exp(-g));
        hrow[r * f + j] = silu * u;
      }
    for (int64_t j = 0; j < f; ++j) {
      for (int64_t c = 0; c < d; ++c) wrow[c] = bf16_to_double(Wd[j * d + c]);
      for (int64_t r = 0; r < nr; ++r) {
        const double hj = hrow[r * f + j];
        double* acc = &yy[r * d];
        for (int64_t c = 0; c < d; ++c) acc[c] += hj * wrow[c];
      }
    }
    for (int64_t r = 0; r < nr; ++r) {
      for (int64_t c = 0; c < d; ++c) y[(r0 + r) * d + c] = yy[r * d + c];
      if (h_out)
        for (int64_t j = 0; j < f; ++j) h_out[(r0 + r) * f + j] = hrow[r * f + j];
    }
  }
  return 0;
}

// Step 6. out[t, c] = sum_j w[t, j] * y_rows[inv_perm[t, j], c] (fp64, j ascending).
int oracle_combine(const double* y_rows, const int32_t* inv_perm, const double* w,
                   int64_t T, int64_t d, int64_t k, double* out) {
  if (!y_rows || !inv_perm || !w || !out || T < 0 || d <= 0 || k <= 0) return 1;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t c = 0; c < d; ++c) out[t * d + c] = 0.0;
    for (int64_t j = 0; j < k; ++j) {
      const double* yr = y_rows + static_cast<int64_t>(inv_perm[t * k + j]) * d;
      const double wj = w[t * k + j];
      for (int64_t c = 0; c < d; ++c) out[t * d + c] += wj * yr[c];
    }
  }
  return 0;
}

// The whole layer for the tokens listed in `tokens` (n_tok of them; all T
// when tokens == NULL): steps 1-3 for those tokens, then step 5 per selected
// (token, expert) pair and step 6. Expert weights are read where they lie
// (bf16, [E, d, 2f] and [E, f, d]) and widened row by row. out is [n_tok, d]
// fp64; idx_out [n_tok, k] and w_out [n_tok, k] may be NULL.
int oracle_forward_tokens(const uint16_t* x, const float* Wr, const float* bias,
                          const uint16_t* Wgu, const uint16_t* Wd,
                          int64_t T, int64_t d, int64_t E, int64_t k, int64_t f,
                          const int64_t* tokens, int64_t n_tok,
                          double* out, int32_t* idx_out, double* w_out) {
  if (!x || !Wr || !Wgu || !Wd || !out || T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E || f <= 0)
    return 1;
  if (!tokens) n_tok = T;
  std::vector<uint16_t> xs(n_tok * d);
  for (int64_t q = 0; q < n_tok; ++q) {
    const int64_t t = tokens ? tokens[q] : q;
    if (t < 0 || t >= T) return 1;
    std::memcpy(&xs[q * d], x + t * d, sizeof(uint16_t) * d);
  }
  std::vector<float> logits(n_tok * E);
  int st = oracle_router_logits(xs.data(), Wr, bias, n_tok, d, E, logits.data());
  if (st) return st;
  std::vector<int32_t> idx(n_tok * k);
  std::vector<double> w(n_tok * k);
  st = oracle_topk(logits.data(), n_tok, E, k, idx.data(), w.data(), nullptr);
  if (st) return st;
  // group the selected pairs by expert so each expert's weights are widened once
  std::vector<int32_t> counts(E), offsets(E + 1), perm_tok(n_tok * k), inv(n_tok * k);
  st = oracle_permute(idx.data(), n_tok, E, k, counts.data(), offsets.data(), perm_tok.data(), inv.data());
  if (st) return st;
  std::vector<double> y(n_tok * k * d);
  const int64_t f2 = 2 * f;
  for (int64_t e = 0; e < E; ++e) {
    const int64_t n = counts[e];
    if (n == 0) continue;
    std::vector<uint16_t> rows(n * d);
    for (int64_t r = 0; r < n; ++r)
      std::memcpy(&rows[r * d], &xs[static_cast<int64_t>(perm_tok[offsets[e] + r]) * d], sizeof(uint16_t) * d);
    st = oracle_expert_ffn(rows.data(), n, Wgu + e * d * f2, Wd + e * f * d, d, f,
                           &y[static_cast<int64_t>(offsets[e]) * d], nullptr);
    if (st) return st;
  }
  st = oracle_combine(y.data(), inv.data(), w.data(), n_tok, d, k, out);
  if (st) return st;
  if (idx_out) std::memcpy(idx_out, idx.data(), sizeof(int32_t) * n_tok * k);
  if (w_out) std::memcpy(w_out, w.data(), sizeof(double) * n_tok * k);
  return 0;
}

// ------------------------------------------------ MXFP4 expert weights
//
// [P3] section "Systems Optimization, Load Balancing, and Post-Training
// Alignment": the MoE weights are served as MXFP4 (with MXFP8 activations).
// The pages do not define the format; reading taken: the published OCP
// Microscaling (MX) format. Blocks of 32 consecutive values along the
// reduction axis share one power-of-two scale 2^s, stored as the unsigned
// 8-bit exponent code s + 127 (E8M0). Each value is a 4-bit E2M1 float: bit 3
// the sign, bits 2..1 an exponent with bias 1, bit 0 a mantissa bit, so the
// magnitudes by 3-bit code are 0, 0.5, 1, 1.5, 2, 3, 4, 6.
// Quantisation, the MX conversion: s = floor(log2(max |v|)) - 2 (2 is the
// exponent of the largest E2M1 magnitude, 6 = 1.5 * 2^2), clamped to
// [-127, 127]; an all-zero block takes s = -127. Each v / 2^s becomes the
// nearest E2M1 magnitude (ties to the even code, whose mantissa bit is 0;
// beyond 6 the nearest is 6, so large values saturate) with the sign of v.
// Dequantised, code c and scale s give (-1)^(c >> 3) * mag[c & 7] * 2^s,
// exactly representable in bf16 for every scale a bf16 block can produce.

namespace {

constexpr int64_t kMxBlock = 32;
const double kE2M1Mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

inline uint8_t e2m1_nearest(double a) {  // a >= 0: code of the nearest magnitude
  int best = 0;
  double bd = std::fabs(a - kE2M1Mag[0]);
  for (int c = 1; c < 8; ++c) {
    const double dist = std::fabs(a - kE2M1Mag[c]);
    if (dist < bd || (dist == bd && (c & 1) == 0)) {
      best = c;
      bd = dist;
    }
  }
  return static_cast<uint8_t>(best);
}

}  // namespace

// w [K, N] bf16 (N contiguous), K % 32 == 0: blocks of 32 along K for each
// column n. codes [K, N] (one E2M1 code per byte), scales [K / 32, N] (E8M0).
int oracle_mxfp4_quantize(const uint16_t* w, int64_t K, int64_t N, uint8_t* codes, uint8_t* scales) {
  if (!w || !codes || !scales || K <= 0 || N <= 0 || K % kMxBlock) return 1;
  for (int64_t b = 0; b < K / kMxBlock; ++b)
    for (int64_t n = 0; n < N; ++n) {
      double amax = 0.0;
      for (int64_t i = 0; i < kMxBlock; ++i) {
        const double v = bf16_to_double(w[(b * kMxBlock + i) * N + n]);
        if (!std::isfinite(v)) return 2;
        amax = std::max(amax, std::fabs(v));
      }
      int s = -127;
      if (amax > 0.0) {
        int e = 0;
        std::frexp(amax, &e);  // amax = m * 2^e, m in [0.5, 1): floor(log2 amax) = e - 1
        s = std::min(127, std::max(-127, e - 1 - 2));
      }
      scales[b * N + n] = static_cast<uint8_t>(s + 127);
      for (int64_t i = 0; i < kMxBlock; ++i) {
        const double v = bf16_to_double(w[(b * kMxBlock + i) * N + n]);
        const uint8_t mag = e2m1_nearest(std::ldexp(std::fabs(v), -s));
        codes[(b * kMxBlock + i) * N + n] = static_cast<uint8_t>((std::signbit(v) ? 8 : 0) | mag);
      }
    }
  return 0;
}

// MXFP8 activations (the same passage): E4M3 elements, the OCP FP8 format
// without infinities: bit 7 the sign, bits 6..3 an exponent with bias 7,
// bits 2..0 a mantissa; magnitude (e == 0 ? m / 8 * 2^-6 : (1 + m / 8) *
// 2^(e - 7)), the largest finite 448 (code 0x7e), 0x7f and 0xff are NaN.
// Blocks of 32 consecutive values along the contiguous (reduction) axis of
// each row share an E8M0 scale 2^s, s = floor(log2(max |v|)) - 8 (8 is the
// exponent of the largest E4M3 magnitude), clamped to [-127, 127]; an
// all-zero block takes s = -127. Each v / 2^s becomes the nearest E4M3
// magnitude (ties to the even code; beyond 448 the nearest is 448, so large
// values saturate) with the sign of v.

namespace {

double e4m3_mag(int c) {  // c in 0..126
  const int e = c >> 3, m = c & 7;
  return e == 0 ? std::ldexp(m / 8.0, -6) : std::ldexp(1.0 + m / 8.0, e - 7);
}

inline uint8_t e4m3_nearest(double a) {  // a >= 0: code of the nearest finite magnitude
  int best = 0;
  double bd = a;
  for (int c = 1; c < 127; ++c) {
    const double dist = std::fabs(a - e4m3_mag(c));
    if (dist < bd || (dist == bd && (c & 1) == 0)) {
      best = c;
      bd = dist;
    }
  }
  return static_cast<uint8_t>(best);
}

}  // namespace

// v [rows, cols] fp64 (cols contiguous), cols % 32 == 0: codes [rows, cols],
// scales [rows, cols / 32].
int oracle_mxfp8_quantize(const double* v, int64_t rows, int64_t cols, uint8_t* codes, uint8_t* scales) {
  if (!v || !codes || !scales || rows <= 0 || cols <= 0 || cols % kMxBlock) return 1;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < cols / kMxBlock; ++b) {
      const double* blk = v + r * cols + b * kMxBlock;
      double amax = 0.0;
      for (int64_t i = 0; i < kMxBlock; ++i) {
        if (!std::isfinite(blk[i])) return 2;
        amax = std::max(amax, std::fabs(blk[i]));
      }
      int s = -127;
      if (amax > 0.0) {
        int e = 0;
        std::frexp(amax, &e);
        s = std::min(127, std::max(-127, e - 1 - 8));
      }
      scales[r * (cols / kMxBlock) + b] = static_cast<uint8_t>(s + 127);
      for (int64_t i = 0; i < kMxBlock; ++i) {
        const uint8_t mag = e4m3_nearest(std::ldexp(std::fabs(blk[i]), -s));
        codes[r * cols + b * kMxBlock + i] = static_cast<uint8_t>((std::signbit(blk[i]) ? 0x80 : 0) | mag);
      }
    }
  return 0;
}

// The inverse, in fp64.
int oracle_mxfp8_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols, double* out) {
  if (!codes || !scales || !out || rows <= 0 || cols <= 0 || cols % kMxBlock) return 1;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t i = 0; i < cols; ++i) {
      const uint8_t c = codes[r * cols + i];
      const uint8_t q = scales[r * (cols / kMxBlock) + i / kMxBlock];
      if ((c & 0x7f) == 0x7f || q == 255) return 1;  // NaN codes
      out[r * cols + i] = (c & 0x80 ? -1.0 : 1.0) * std::ldexp(e4m3_mag(c & 0x7f), static_cast<int>(q) - 127);
    }
  return 0;
}

// The expert feed-forward of step 5 with MXFP8 activations and MXFP4 weights
// (the serving format above): x_mx [n, d] are the rows after their MXFP8
// round trip (fp64), Wgu [d, 2f] and Wd [f, d] the dequantised MXFP4 weights
// (bf16 bits, exact). g, u and h = SiLU(g) * u as in step 5 (fp64); h, the
// down projection's activation operand, takes its own MXFP8 round trip along
// f before y = h' Wd. h_out (may be NULL) receives h'. f % 32 == 0.
int oracle_expert_ffn_mx(const double* x_mx, int64_t n, const uint16_t* Wgu, const uint16_t* Wd, int64_t d,
                         int64_t f, double* y, double* h_out) {
  if ((!x_mx && n > 0) || !Wgu || !Wd || !y || n < 0 || d <= 0 || f <= 0 || f % kMxBlock) return 1;
  const int64_t f2 = 2 * f;
  int status = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < n; ++r) {
    std::vector<double> gu(f2, 0.0), hrow(f), yy(d, 0.0);
    std::vector<uint8_t> hc(f), hs(f / kMxBlock);
    for (int64_t i = 0; i < d; ++i) {
      const double xi = x_mx[r * d + i];
      for (int64_t j = 0; j < f2; ++j) gu[j] += xi * bf16_to_double(Wgu[i * f2 + j]);
    }
    for (int64_t j = 0; j < f; ++j) {
      const double g = gu[j], u = gu[f + j];
      hrow[j] = g / (1.0 + std::exp(-g)) * u;
    }
    int st = oracle_mxfp8_quantize(hrow.data(), 1, f, hc.data(), hs.data());
    if (!st) st = oracle_mxfp8_dequantize(hc.data(), hs.data(), 1, f, hrow.data());
    if (st) {
#pragma omp critical
      status = st;
      continue;
    }
    for (int64_t j = 0; j < f; ++j) {
      const double hj = hrow[j];
      for (int64_t c = 0; c < d; ++c) yy[c] += hj * bf16_to_double(Wd[j * d + c]);
    }
    for (int64_t c = 0; c < d; ++c) y[r * d + c] = yy[c];
    if (h_out)
      for (int64_t j = 0; j < f; ++j) h_out[r * f + j] = hrow[j];
  }
  return status;
}

// The inverse: w_out [K, N] as bf16 bits (every value is exact in bf16).
int oracle_mxfp4_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t K, int64_t N, uint16_t* w_out) {
  if (!codes || !scales || !w_out || K <= 0 || N <= 0 || K % kMxBlock) return 1;
  for (int64_t r = 0; r < K; ++r)
    for (int64_t n = 0; n < N; ++n) {
      const uint8_t c = codes[r * N + n];
      if (c > 15 || scales[(r / kMxBlock) * N + n] == 255) return 1;  // 255: the E8M0 NaN
      const int s = static_cast<int>(scales[(r / kMxBlock) * N + n]) - 127;
      const double v = (c & 8 ? -1.0 : 1.0) * std::ldexp(kE2M1Mag[c & 7], s);
      const float fv = static_cast<float>(v);  // exact: at most two significant bits
      uint32_t u;
      std::memcpy(&u, &fv, sizeof(u));
      w_out[r * N + n] = static_cast<uint16_t>(u >> 16);
    }
  return 0;
}

}  // extern "C"

// ------------------------------------------------ Quantile Balancing
//
// [P3] section "Systems Optimization, Load Balancing, and Post-Training
// Alignment": Quantile Balancing (QB) sets the router's per-expert biases from
// the dual of the balanced-assignment linear program. For m tokens, n experts,
// top-k routing and target load q = m k / n, each expert's bias comes from the
// (1 - k/n)-quantile, over tokens, of the margins s[i,j] - alpha_i, where
// alpha_i is token i's cutoff under top-(k+1) routing. The update formula
// itself is missing from the page; reading taken, from that LP:
//   maximise sum s[i,j] x[i,j]  s.t.  sum_j x[i,j] = k,  sum_i x[i,j] <= q,
//   0 <= x <= 1,
// whose dual has a price alpha_i per token and beta_j per expert. With the
// current biases b (b = -beta), alpha_i is the (k+1)-th largest of
// s[i,j] + b_j (the best biased score left out of the top k), and the beta_j
// minimising the dual objective q beta_j + sum_i max(0, s[i,j] - alpha_i -
// beta_j) for that alpha is the ceil(q)-th largest margin s[i,j] - alpha_i
// over tokens: the (1 - k/n)-quantile. The new bias is b_j = -beta_j. The
// scores s are the router logits, the quantity the bias shifts.
// Histogram form (the page's per-expert binned counts H[n][B], B = 1000 there,
// summed over data-parallel ranks by one integer all-reduce): the margins of
// expert j are counted in B equal bins over [lo, hi) (the range is not given
// on the page: a parameter here), a margin below lo in bin 0 and one at or
// above hi in bin B - 1. beta_j is then the lower edge of the bin that holds
// the ceil(q)-th largest margin, within one bin width (hi - lo) / B of the
// exact value when every margin lies in [lo, hi).

namespace {

// ceil(m k / n) clamped to [1, m]: the rank, from the top, of the quantile.
int64_t qb_rank(int64_t m, int64_t n, int64_t k) {
  int64_t r = (m * k + n - 1) / n;
  return std::max<int64_t>(1, std::min(r, m));
}

}  // namespace

extern "C" {

// alpha[i] = (k+1)-th largest of s[i,j] + b[j] over j (b may be NULL: zero).
// s [m, n] row-major. 1 <= k < n.
int oracle_qb_cutoffs(const double* s, const double* b, int64_t m, int64_t n, int64_t k, double* alpha) {
  if (!s || !alpha || m < 1 || n < 2 || k < 1 || k >= n) return 1;
  std::vector<double> v(n);
  for (int64_t i = 0; i < m; ++i) {
    for (int64_t j = 0; j < n; ++j) v[j] = s[i * n + j] + (b ? b[j] : 0.0);
    std::nth_element(v.begin(), v.begin() + k, v.end(), std::greater<double>());
    alpha[i] = v[k];
  }
  return 0;
}

// One QB step with exact quantiles: b_new[j] = -(ceil(m k / n)-th largest of
// s[i,j] - alpha[i] over i), alpha from oracle_qb_cutoffs(s, b).
int oracle_qb_update(const double* s, const double* b, int64_t m, int64_t n, int64_t k, double* b_new) {
  if (!b_new) return 1;
  std::vector<double> alpha(m > 0 ? m : 1);
  const int st = oracle_qb_cutoffs(s, b, m, n, k, alpha.data());
  if (st) return st;
  const int64_t r = qb_rank(m, n, k);
  std::vector<double> mu(m);
  for (int64_t j = 0; j < n; ++j) {
    for (int64_t i = 0; i < m; ++i) mu[i] = s[i * n + j] - alpha[i];
    std::nth_element(mu.begin(), mu.begin() + (r - 1), mu.end(), std::greater<double>());
    b_new[j] = -mu[r - 1];
  }
  return 0;
}

// H[j][bin] += 1 for each token's margin s[i,j] - alpha[i] (H [n, B] int64,
// accumulated into, so several batches or ranks can add up).
int oracle_qb_histogram(const double* s, const double* alpha, int64_t m, int64_t n, double lo, double hi, int64_t B,
                        int64_t* H) {
  if (!s || !alpha || !H || m < 0 || n < 1 || B < 1 || !(hi > lo)) return 1;
  for (int64_t i = 0; i < m; ++i)
    for (int64_t j = 0; j < n; ++j) {
      const double mu = s[i * n + j] - alpha[i];
      // bin floor(B (mu - lo) / (hi - lo)): exact on the edges that exact
      // inputs put there (a margin of 0 -- the cutoff expert's own -- with lo
      // a multiple of the bin width), where dividing by a rounded width is not
      // (a NaN margin fails mu >= lo and counts in bin 0, as below lo)
      int64_t bin =
          !(mu >= lo) ? 0 : static_cast<int64_t>(std::floor(static_cast<double>(B) * (mu - lo) / (hi - lo)));
      bin = std::max<int64_t>(0, std::min(bin, B - 1));
      H[j * B + bin] += 1;
    }
  return 0;
}

// b_new[j] = -(lower edge of the bin of H[j] holding the ceil(m_total k / n)-th
// largest margin), m_total the number of tokens counted in each row of H.
int oracle_qb_bias_from_histogram(const int64_t* H, int64_t n, int64_t B, double lo, double hi, int64_t m_total,
                                  int64_t k, double* b_new) {
  if (!H || !b_new || n < 2 || B < 1 || !(hi > lo) || m_total < 1 || k < 1 || k >= n) return 1;
  const int64_t r = qb_rank(m_total, n, k);
  const double width = (hi - lo) / static_cast<double>(B);
  for (int64_t j = 0; j < n; ++j) {
    int64_t total = 0;
    for (int64_t t = 0; t < B; ++t) total += H[j * B + t];
    if (total != m_total) return 2;  // every token is counted once per expert
    int64_t c = 0, bin = B - 1;
    for (; bin > 0; --bin) {
      c += H[j * B + bin];
      if (c >= r) break;
    }
    b_new[j] = -(lo + static_cast<double>(bin) * width);
  }
  return 0;
}

}  // extern "C"

extern "C" {

// The histogram with the decisions taken in fp32, as a GPU computing on fp32
// router logits takes them: v = s + b rounded to fp32, alpha the (k+1)-th
// largest v, mu = s - alpha rounded to fp32, t = mu - lo rounded to fp32, and
// the bin floor(t * inv_w) with inv_w = fp32(B) / fp32(hi - lo), both
// products rounded to fp32; t < 0 (or NaN) counts in bin 0, a bin >= B in
// bin B - 1.
// On data with no margin within an fp32 rounding of a bin edge it counts
// exactly what oracle_qb_histogram counts (from the same fp32 inputs).
// s [m, n] fp32, b [n] fp32 or NULL; alpha [m] (fp32 values) is written.
int oracle_qb_histogram_f32(const float* s, const float* b, int64_t m, int64_t n, int64_t k, float lo, float hi,
                            int64_t B, float* alpha, int64_t* H) {
  if (!s || !alpha || !H || m < 1 || n < 2 || k < 1 || k >= n || B < 1 || !(hi > lo)) return 1;
  const float inv_w = static_cast<float>(B) / (hi - lo);
  std::vector<float> v(n);
  for (int64_t i = 0; i < m; ++i) {
    for (int64_t j = 0; j < n; ++j) v[j] = s[i * n + j] + (b ? b[j] : 0.0f);
    std::nth_element(v.begin(), v.begin() + k, v.end(), std::greater<float>());
    alpha[i] = v[k];
    for (int64_t j = 0; j < n; ++j) {
      const float mu = s[i * n + j] - alpha[i];
      const float t = mu - lo;
      const float fbin = t * inv_w;
      int64_t bin = !(t >= 0.0f) ? 0 : (fbin >= static_cast<float>(B) ? B - 1 : static_cast<int64_t>(fbin));
      H[j * B + bin] += 1;
    }
  }
  return 0;
}

// The quantile's bin per expert: bins[j] = the bin of H[j] holding the
// ceil(m_total k / n)-th largest margin (the integer half of
// oracle_qb_bias_from_histogram).
int oracle_qb_quantile_bins(const int64_t* H, int64_t n, int64_t B, int64_t m_total, int64_t k, int64_t* bins) {
  if (!H || !bins || n < 2 || B < 1 || m_total < 1 || k < 1 || k >= n) return 1;
  const int64_t r = qb_rank(m_total, n, k);
  for (int64_t j = 0; j < n; ++j) {
    int64_t c = 0, bin = B - 1;
    for (; bin > 0; --bin) {
      c += H[j * B + bin];
      if (c >= r) break;
    }
    bins[j] = bin;
  }
  return 0;
}

}  // extern "C"

// ------------------------------------------------ Stable LatentMoE (next row)
//
// [P3] section "Operational Execution Flow": two full-width shared experts act
// on x directly; the routed path projects x down to a latent z = x W_dn of
// width l (3584 on the page); the k active routed experts act on z; their
// probability-weighted sum u = sum_{i in top-k} p_i E_i(z) passes an explicit
// RMSNorm and W_up brings it back to width d. The experts' GLU is SiTU-GLU
// ("Sigmoid Tanh Unit GLU"), a soft-capped SwiGLU with beta1 = 4, beta2 = 25,
// for which the page states |SiTU-GLU| <= beta1 beta2 = 100. The page's
// formulas for SiTU-GLU and for the layer output did not survive. Readings:
//   SiTU-GLU(g, v) = beta1 tanh(SiLU(g) / beta1) * beta2 tanh(v / beta2):
//     SiLU's sigmoid, a tanh soft cap on each factor, so the product is
//     bounded by beta1 beta2, and it equals SwiGLU's SiLU(g) v wherever
//     |SiLU(g)| << beta1 and |v| << beta2 (SwiGLU's linear regime);
//   out = sum_s S_s(x) + RMSNorm(u) W_up, RMSNorm(u) = gamma u / sqrt(mean(u^2) + eps);
//   the router reads x (width d), as the plain layer's does; no biases.
// SiTU-GLU's own formula is therefore parity-unpinned: what pins it is the
// stated bound, its limit SwiGLU as beta1, beta2 -> infinity, and the layer's
// reduction to the RMSNorm of the plain layer.

namespace {

inline double silu(double a) { return a / (1.0 + std::exp(-a)); }

// act 0: SwiGLU SiLU(g) v; act 1: SiTU-GLU with caps b1, b2.
inline double glu(double g, double v, int act, double b1, double b2) {
  if (act == 0) return silu(g) * v;
  return b1 * std::tanh(silu(g) / b1) * (b2 * std::tanh(v / b2));
}

}  // namespace

extern "C" {

// One GLU feed-forward on fp64 rows: x [n, K], W_gu [K, 2F] (columns 0..F-1
// gate, F..2F-1 the second factor), W_d [F, N], bf16 weights; y [n, N] fp64;
// h (optional) [n, F] the activation. act 0 SwiGLU, 1 SiTU-GLU (b1, b2).
int oracle_glu_ffn(const double* x, int64_t n, const uint16_t* Wgu, const uint16_t* Wd, int64_t K, int64_t F,
                   int64_t N, int act, double b1, double b2, double* y, double* h_out) {
  if ((!x && n > 0) || !Wgu || !Wd || !y || n < 0 || K <= 0 || F <= 0 || N <= 0 || (act != 0 && act != 1))
    return 1;
  if (act == 1 && !(b1 > 0.0 && b2 > 0.0)) return 1;
  const int64_t F2 = 2 * F;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < n; ++r) {
    std::vector<double> gv(F2, 0.0), h(F), yy(N, 0.0);
    for (int64_t i = 0; i < K; ++i) {
      const double xi = x[r * K + i];
      for (int64_t j = 0; j < F2; ++j) gv[j] += xi * bf16_to_double(Wgu[i * F2 + j]);
    }
    for (int64_t j = 0; j < F; ++j) h[j] = glu(gv[j], gv[F + j], act, b1, b2);
    for (int64_t j = 0; j < F; ++j)
      for (int64_t c = 0; c < N; ++c) yy[c] += h[j] * bf16_to_double(Wd[j * N + c]);
    for (int64_t c = 0; c < N; ++c) y[r * N + c] = yy[c];
    if (h_out)
      for (int64_t j = 0; j < F; ++j) h_out[r * F + j] = h[j];
  }
  return 0;
}

// RMSNorm of each row: out = gamma * u / sqrt(mean(u^2) + eps); gamma [l]
// fp32 or NULL (ones). u, out [n, l] fp64 (may alias).
int oracle_rmsnorm(const double* u, int64_t n, int64_t l, const float* gamma, double eps, double* out) {
  if ((!u && n > 0) || !out || n < 0 || l <= 0 || !(eps >= 0.0)) return 1;
  for (int64_t r = 0; r < n; ++r) {
    double ss = 0.0;
    for (int64_t c = 0; c < l; ++c) ss += u[r * l + c] * u[r * l + c];
    const double den = std::sqrt(ss / static_cast<double>(l) + eps);
    for (int64_t c = 0; c < l; ++c)
      out[r * l + c] = (gamma ? static_cast<double>(gamma[c]) : 1.0) * (den > 0.0 ? u[r * l + c] / den : 0.0);
  }
  return 0;
}

// The Stable LatentMoE layer for T tokens (readings above). x [T, d] bf16;
// W_router [d, E] fp32, bias [E] or NULL; W_dn [d, l] and W_up [l, d] bf16;
// routed experts W_gu [E, l, 2f], W_d [E, f, l] bf16; gamma [l] fp32 or NULL;
// shared experts Ws_gu [S, d, 2fs], Ws_d [S, fs, d] bf16 (S may be 0); act,
// b1, b2 the experts' GLU; eps the RMSNorm's. out [T, d] fp64; u_out
// (optional) [T, l] the routed sum before the RMSNorm.
int oracle_latent_forward(const uint16_t* x, const float* Wr, const float* bias, const uint16_t* Wdn,
                          const uint16_t* Wup, const uint16_t* Wgu, const uint16_t* Wd, const float* gamma,
                          const uint16_t* Wsgu, const uint16_t* Wsd, int64_t T, int64_t d, int64_t l, int64_t E,
                          int64_t k, int64_t f, int64_t S, int64_t fs, int act, double b1, double b2, double eps,
                          double* out, double* u_out) {
  if (!x || !Wr || !Wdn || !Wup || !Wgu || !Wd || !out || T < 0 || d <= 0 || l <= 0 || E <= 0 || k <= 0 || k > E ||
      f <= 0 || S < 0 || (S > 0 && (!Wsgu || !Wsd || fs <= 0)))
    return 1;
  // 1-3. route on x
  std::vector<float> logits(T * E);
  int st = oracle_router_logits(x, Wr, bias, T, d, E, logits.data());
  if (st) return st;
  std::vector<int32_t> idx(T * k);
  std::vector<double> w(T * k);
  st = oracle_topk(logits.data(), T, E, k, idx.data(), w.data(), nullptr);
  if (st) return st;
  // z = x W_dn (fp64)
  std::vector<double> xd(T * d), z(T * l, 0.0);
  for (int64_t q = 0; q < T * d; ++q) xd[q] = bf16_to_double(x[q]);
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t)
    for (int64_t i = 0; i < d; ++i) {
      const double xi = xd[t * d + i];
      for (int64_t c = 0; c < l; ++c) z[t * l + c] += xi * bf16_to_double(Wdn[i * l + c]);
    }
  // routed experts on z, rows grouped by expert; u = sum_j p_j E_j(z) in slot order
  std::vector<int32_t> counts(E), offsets(E + 1), perm(T * k), inv(T * k);
  st = oracle_permute(idx.data(), T, E, k, counts.data(), offsets.data(), perm.data(), inv.data());
  if (st) return st;
  std::vector<double> y(T * k * l);
  for (int64_t e = 0; e < E; ++e) {
    const int64_t n = counts[e];
    if (n == 0) continue;
    std::vector<double> rows(n * l);
    for (int64_t r = 0; r < n; ++r)
      std::memcpy(&rows[r * l], &z[static_cast<int64_t>(perm[offsets[e] + r]) * l], sizeof(double) * l);
    st = oracle_glu_ffn(rows.data(), n, Wgu + e * l * 2 * f, Wd + e * f * l, l, f, l, act, b1, b2,
                        &y[static_cast<int64_t>(offsets[e]) * l], nullptr);
    if (st) return st;
  }
  std::vector<double> u(T * l, 0.0);
  for (int64_t t = 0; t < T; ++t)
    for (int64_t j = 0; j < k; ++j) {
      const double* yr = &y[static_cast<int64_t>(inv[t * k + j]) * l];
      for (int64_t c = 0; c < l; ++c) u[t * l + c] += w[t * k + j] * yr[c];
    }
  if (u_out) std::memcpy(u_out, u.data(), sizeof(double) * T * l);
  // RMSNorm, then W_up back to width d
  std::vector<double> un(T * l);
  st = oracle_rmsnorm(u.data(), T, l, gamma, eps, un.data());
  if (st) return st;
  for (int64_t q = 0; q < T * d; ++q) out[q] = 0.0;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t)
    for (int64_t c = 0; c < l; ++c) {
      const double v = un[t * l + c];
      for (int64_t o = 0; o < d; ++o) out[t * d + o] += v * bf16_to_double(Wup[c * d + o]);
    }
  // shared experts on x, added after
  std::vector<double> ys(T * d);
  for (int64_t s = 0; s < S; ++s) {
    st = oracle_glu_ffn(xd.data(), T, Wsgu + s * d * 2 * fs, Wsd + s * fs * d, d, fs, d, act, b1, b2, ys.data(),
                        nullptr);
    if (st) return st;
    for (int64_t q = 0; q < T * d; ++q) out[q] += ys[q];
  }
  return 0;
}

}  // extern "C"
