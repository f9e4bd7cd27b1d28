// fp64 CPU oracle of the predictor-gated sparse FFN -- TEST INFRASTRUCTURE.
//
// A plain, slow, single-threaded C++ program: explicit loops over fp64
// values, no BLAS, no blocking, no threads.  Only the test suite, the package
// smoke check and the benchmark's CPU-baseline and reference legs load it
// (through oracle/cpp.py); the CUDA library never calls it and shares no code,
// header, table or constant with it.
//
// What it computes, and where the pages state it (PowerInfer):
//   * Per token and layer a predictor scores every FFN neuron; only neurons
//     predicted active are processed, the rest are skipped (unite.ai page,
//     "Adaptive Sparsity-Prädiktoren"; machine-heart page, Figure 8: the
//     prediction decides, a neuron labelled hot but predicted inactive is
//     skipped).
//   * The active neurons form a table mapping each neuron to its original
//     weight row (unite.ai page, "Neuronen-Platzierung und -Verwaltung").
//   * The neuron-aware operator computes only those neurons' row vectors of
//     W_up (and W_gate) and of W_down^T, with no sparse-format conversion
//     (unite.ai page, "Neuronenbewusster Operator").
//   * ReLU, ReGLU and Squared-ReLU models; INT4 Q4_0 weights (GeekNews page,
//     summary, limitations list and quantisation notes).
//
// The pages give no formulas; the readings taken (each stated where it is
// used below):
//   predictor   a = relu(W1 x + b1), s = W2 a + b2, active iff s > tau
//               (a tie is inactive);
//   batch       the active set is the ascending union of the tokens' sets and
//               every token is computed on the whole union;
//   neurons     ReLU h = max(W_up[i].x + b_up[i], 0);
//               ReGLU h = max(W_gate[i].x + b_gate[i], 0) * (W_up[i].x);
//               Squared-ReLU h = max(W_up[i].x + b_up[i], 0)^2;
//   output      y = sum over listed i of h_i W_down^T[i] (no down bias);
//   stack       x_l = round16(x / sqrt(mean(x^2) + 1e-6)), x += FFN(x_l);
//   Q4_0        per 32-element block an fp16 scale then 16 bytes, byte j
//               holding element j (low nibble) and j + 16 (high nibble);
//               value = (q - 8) * scale.
// Every stored weight is widened exactly to fp64 from its bit fields; every
// operation after that is an fp64 multiply, add, max, divide or square root.
#include <cmath>
#include <cstddef>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

// ------------------------------------------------------------ widening
// IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
double widen_f16_bits(uint16_t b) {
  const int sign = b >> 15;
  const int e = (b >> 10) & 0x1f;
  const int m = b & 0x3ff;
  double v;
  if (e == 0) {
    v = std::ldexp((double)m, -24);  // subnormal: m * 2^-24
  } else if (e == 31) {
    v = m ? std::nan("") : INFINITY;
  } else {
    v = std::ldexp((double)(1024 + m), e - 25);  // (1 + m/2^10) * 2^(e-15)
  }
  return sign ? -v : v;
}

// bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits.
double widen_bf16_bits(uint16_t b) {
  const int sign = b >> 15;
  const int e = (b >> 7) & 0xff;
  const int m = b & 0x7f;
  double v;
  if (e == 0) {
    v = std::ldexp((double)m, -133);  // subnormal: m * 2^-133
  } else if (e == 255) {
    v = m ? std::nan("") : INFINITY;
  } else {
    v = std::ldexp((double)(128 + m), e - 134);  // (1 + m/2^7) * 2^(e-127)
  }
  return sign ? -v : v;
}

// One Q4_0 row (d/32 blocks of 18 bytes) -> d fp64 values.
void dequant_q4_0_row(const uint8_t* row, int d, double* out) {
  for (int blk = 0; blk < d / 32; ++blk) {
    const uint8_t* p = row + (size_t)blk * 18;
    const double scale = widen_f16_bits((uint16_t)(p[0] | (p[1] << 8)));  // little endian
    for (int j = 0; j < 16; ++j) {
      const int lo = p[2 + j] & 0x0f;
      const int hi = p[2 + j] >> 4;
      out[blk * 32 + j] = (double)(lo - 8) * scale;
      out[blk * 32 + j + 16] = (double)(hi - 8) * scale;
    }
  }
}

// The value of every 16-bit pattern, decoded once by the functions above, so
// that widening a row is one table read per element.
const std::vector<double>& pattern_values(int dtype) {
  static const std::vector<double> f16 = [] {
    std::vector<double> t(65536);
    for (int b = 0; b < 65536; ++b) t[b] = widen_f16_bits((uint16_t)b);
    return t;
  }();
  static const std::vector<double> bf16 = [] {
    std::vector<double> t(65536);
    for (int b = 0; b < 65536; ++b) t[b] = widen_bf16_bits((uint16_t)b);
    return t;
  }();
  return dtype == 0 ? f16 : bf16;
}

// dtype codes: 0 fp16, 1 bf16, 2 Q4_0
void widen_row(const void* base, int dtype, int64_t row, int d, double* out) {
  if (dtype == 2) {
    dequant_q4_0_row(static_cast<const uint8_t*>(base) + (size_t)row * (d / 32) * 18, d, out);
    return;
  }
  const uint16_t* p = static_cast<const uint16_t*>(base) + (size_t)row * d;
  const double* v = pattern_values(dtype).data();
  for (int k = 0; k < d; ++k) out[k] = v[p[k]];
}

// ------------------------------------------------------------ rounding
// Round to nearest, ties to even, to a binary format with `sig` significand
// bits (hidden bit included), minimum normal exponent emin (of the value
// 1.xxx * 2^E) and largest finite value `maxv`.  One rounding from fp64.
double round_fmt(double x, int sig, int emin, double maxv) {
  if (x == 0.0 || std::isnan(x) || std::isinf(x)) return x;
  const double ax = std::fabs(x);
  // halfway between maxv and the next (unrepresentable) value rounds to even,
  // which is the overflow value: anything at or above it is infinite
  const double ovf = maxv + std::ldexp(1.0, std::ilogb(maxv) - sig);
  if (ax >= ovf) return std::copysign(INFINITY, x);
  int E = std::ilogb(ax);                 // ax = 1.f * 2^E
  if (E < emin) E = emin;                 // subnormal range: fixed quantum
  const int qe = E - (sig - 1);           // weight of the last significand bit
  const double q = std::nearbyint(std::ldexp(ax, -qe));  // default mode: ties to even
  return std::copysign(std::ldexp(q, qe), x);
}

double round_f16(double x) { return round_fmt(x, 11, -14, 65504.0); }
double round_bf16(double x) {
  return round_fmt(x, 8, -126, std::ldexp(255.0, 120));  // (2 - 2^-7) * 2^127
}
double round16(double x, int adtype) { return adtype == 0 ? round_f16(x) : round_bf16(x); }

}  // namespace

extern "C" {

// Layer descriptor: host pointers to the stored weights (bits exactly as the
// GPU reads them) and fp64 copies of the fp32 biases.
struct po_layer {
  int32_t d_model, d_ff, rank;
  int32_t act;     // 0 ReLU, 1 ReGLU, 2 Squared-ReLU
  int32_t wdtype;  // FFN matrices: 0 fp16, 1 bf16, 2 Q4_0
  int32_t pdtype;  // predictor matrices: 0 fp16, 1 bf16
  const void* w1;  // [rank x d]
  const double* b1;  // [rank] or null
  const void* w2;  // [d_ff x rank]
  const double* b2;  // [d_ff]
  double threshold;
  const void* w_up;      // [d_ff x d] rows
  const void* w_gate;    // ReGLU only
  const void* w_down_t;  // [d_ff x d] rows
  const double* b_up;    // [d_ff] or null (ReLU, Squared-ReLU)
  const double* b_gate;  // [d_ff] or null (ReGLU)
};

double po_widen_f16(uint16_t bits) { return widen_f16_bits(bits); }
double po_widen_bf16(uint16_t bits) { return widen_bf16_bits(bits); }

void po_widen_f16_n(const uint16_t* bits, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = widen_f16_bits(bits[i]);
}
void po_widen_bf16_n(const uint16_t* bits, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = widen_bf16_bits(bits[i]);
}
void po_dequant_q4_0(const uint8_t* rows, int64_t n_rows, int32_t d_model, double* out) {
  for (int64_t r = 0; r < n_rows; ++r)
    dequant_q4_0_row(rows + (size_t)r * (d_model / 32) * 18, d_model, out + (size_t)r * d_model);
}

void po_round_f16_n(const double* x, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = round_f16(x[i]);
}
void po_round_bf16_n(const double* x, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = round_bf16(x[i]);
}

// Layer input of the stack (reading: pre-norm residual chain):
// out = round16(x / sqrt(mean(x^2) + 1e-6)) per token, x [B x d].
void po_rms_cast(const double* x, int32_t B, int32_t d, int32_t adtype, double* out) {
  for (int b = 0; b < B; ++b) {
    const double* xb = x + (size_t)b * d;
    double ss = 0.0;
    for (int k = 0; k < d; ++k) ss += xb[k] * xb[k];
    const double rms = std::sqrt(ss / d + 1e-6);
    for (int k = 0; k < d; ++k) out[(size_t)b * d + k] = round16(xb[k] / rms, adtype);
  }
}

// Predictor (unite.ai page, "Adaptive Sparsity-Prädiktoren"): for tokens x
// [B x d], a [B x r] = relu(W1 x + b1), s [B x F] = W2 a + b2,
// mask [B x F] = s > threshold (1/0).
void po_predict(const po_layer* L, const double* x, int32_t B, double* a, double* s,
                uint8_t* mask) {
  const int d = L->d_model, r = L->rank, F = L->d_ff;
  std::vector<double> w(d > r ? d : r), z(B);
  // Each token's dot product is summed in index order; the tokens are
  // interleaved (x and a held index-major) only so that their independent
  // sums overlap in time.
  std::vector<double> xt((size_t)d * B), at((size_t)r * B);
  for (int b = 0; b < B; ++b)
    for (int k = 0; k < d; ++k) xt[(size_t)k * B + b] = x[(size_t)b * d + k];
  for (int j = 0; j < r; ++j) {
    widen_row(L->w1, L->pdtype, j, d, w.data());
    for (int b = 0; b < B; ++b) z[b] = 0.0;
    for (int k = 0; k < d; ++k)
      for (int b = 0; b < B; ++b) z[b] += w[k] * xt[(size_t)k * B + b];
    for (int b = 0; b < B; ++b) {
      if (L->b1) z[b] += L->b1[j];
      a[(size_t)b * r + j] = z[b] > 0.0 ? z[b] : 0.0;
      at[(size_t)j * B + b] = a[(size_t)b * r + j];
    }
  }
  for (int n = 0; n < F; ++n) {
    widen_row(L->w2, L->pdtype, n, r, w.data());
    for (int b = 0; b < B; ++b) z[b] = 0.0;
    for (int j = 0; j < r; ++j)
      for (int b = 0; b < B; ++b) z[b] += w[j] * at[(size_t)j * B + b];
    for (int b = 0; b < B; ++b) {
      z[b] += L->b2[n];
      s[(size_t)b * F + n] = z[b];
      mask[(size_t)b * F + n] = z[b] > L->threshold ? 1 : 0;
    }
  }
}

// Neuron table (unite.ai page, "Neuronen-Platzierung und -Verwaltung"): the
// ascending list of neurons whose mask is set for at least one token.
// Returns K, the list length.
int64_t po_union_index(const uint8_t* mask, int32_t B, int32_t F, int64_t* idx) {
  int64_t K = 0;
  for (int n = 0; n < F; ++n) {
    bool any = false;
    for (int b = 0; b < B; ++b) any = any || mask[(size_t)b * F + n] != 0;
    if (any) idx[K++] = n;
  }
  return K;
}

// Neurons whose logit lies within `width` of the threshold (either decision
// is correct there for a rounding-level difference in s).
void po_band(const double* s, int64_t n, double threshold, double width, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = std::fabs(s[i] - threshold) < width ? 1 : 0;
}

// h [B x K]: the activation of each listed neuron for each token (unite.ai
// page, "Neuronenbewusster Operator": one weight row per active neuron).
// Returns 0, or -1 if a listed id lies outside [0, d_ff).
int32_t po_neuron_outputs(const po_layer* L, const double* x, int32_t B, const int64_t* idx,
                          int64_t K, double* h) {
  const int d = L->d_model;
  std::vector<double> up(d), gate(d), u(B), g(B), xt((size_t)d * B);
  for (int b = 0; b < B; ++b)  // x held index-major (see po_predict)
    for (int c = 0; c < d; ++c) xt[(size_t)c * B + b] = x[(size_t)b * d + c];
  for (int64_t k = 0; k < K; ++k) {
    const int64_t i = idx[k];
    if (i < 0 || i >= L->d_ff) return -1;
    widen_row(L->w_up, L->wdtype, i, d, up.data());
    if (L->act == 1) widen_row(L->w_gate, L->wdtype, i, d, gate.data());
    // per token, the dot products are summed in index order
    for (int b = 0; b < B; ++b) u[b] = g[b] = 0.0;
    for (int c = 0; c < d; ++c)
      for (int b = 0; b < B; ++b) u[b] += up[c] * xt[(size_t)c * B + b];
    if (L->act == 1)
      for (int c = 0; c < d; ++c)
        for (int b = 0; b < B; ++b) g[b] += gate[c] * xt[(size_t)c * B + b];
    for (int b = 0; b < B; ++b) {
      double v;
      if (L->act == 1) {  // ReGLU: relu(gate pre-activation) * up projection
        double gb = g[b];
        if (L->b_gate) gb += L->b_gate[i];
        v = (gb > 0.0 ? gb : 0.0) * u[b];
      } else {
        double ub = u[b];
        if (L->b_up) ub += L->b_up[i];
        const double rl = ub > 0.0 ? ub : 0.0;
        v = L->act == 2 ? rl * rl : rl;  // Squared-ReLU squares the ReLU output
      }
      h[(size_t)b * K + k] = v;
    }
  }
  return 0;
}

// y [B x d] = sum over the listed neurons i (in list order) of
// h_i * W_down^T[i].  Returns 0, or -1 for an id outside [0, d_ff).
int32_t po_masked_ffn(const po_layer* L, const double* x, int32_t B, const int64_t* idx,
                      int64_t K, double* y) {
  const int d = L->d_model;
  for (size_t e = 0; e < (size_t)B * d; ++e) y[e] = 0.0;
  if (K == 0) return 0;
  std::vector<double> h((size_t)B * K), row(d);
  if (po_neuron_outputs(L, x, B, idx, K, h.data())) return -1;
  for (int64_t k = 0; k < K; ++k) {
    widen_row(L->w_down_t, L->wdtype, idx[k], d, row.data());
    for (int b = 0; b < B; ++b) {
      const double hb = h[(size_t)b * K + k];
      double* yb = y + (size_t)b * d;
      for (int c = 0; c < d; ++c) yb[c] += hb * row[c];
    }
  }
  return 0;
}

// One layer of the method: predict, take the union, compute the masked FFN.
// y [B x d], idx [d_ff] (first K valid), s [B x d_ff].  Returns K.
int64_t po_sparse_ffn_layer(const po_layer* L, const double* x, int32_t B, double* y,
                            int64_t* idx, double* s) {
  std::vector<double> a((size_t)B * L->rank);
  std::vector<uint8_t> mask((size_t)B * L->d_ff);
  po_predict(L, x, B, a.data(), s, mask.data());
  const int64_t K = po_union_index(mask.data(), B, L->d_ff, idx);
  po_masked_ffn(L, x, B, idx, K, y);
  return K;
}

}  // extern "C"
