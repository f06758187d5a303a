// fp64 CPU oracle for the bidirectional multi-head self-attention core of a
// ViT / SigLIP vision encoder.  TEST INFRASTRUCTURE ONLY: the tests, the smoke
// check and the benchmark's CPU-baseline leg call it; the CUDA library never
// does, and it shares no code, header or constant with the CUDA path.
//
// What it computes (the plain definition, written out with no tiling, no
// fusion and no reordering):
//
//   for every image b, head h and query token i:
//     s_j  = scale * sum_c q[b,i,h,c] * k[b,j,h,c]          j = 0..N-1
//     m    = max_j s_j
//     p_j  = exp(s_j - m)
//     l    = sum_j p_j
//     o[b,i,h,c] = (sum_j p_j * v[b,j,h,c]) / l
//
// Sources:
//  * "Pi0 VLA deployment tutorial: Flash Attention for the vision encoder",
//    section 1: the encoder's time goes to the multi-head self-attention
//    layers of the ViT backbone, and Flash Attention changes only the memory
//    access pattern, not the output quality -- so the fused kernel must reach
//    this same result up to rounding.
//  * Same page, section 3.2: the ViT block's qkv linear feeds the attention
//    module (nn.MultiheadAttention swapped for FlashMHA); every patch token and
//    the CLS token attend to every token (bidirectional, no mask), dropout is
//    the inference value 0.
//  * "Pi0 VLA latency report on a 16 GB GPU", section 3.1: ViT-L/14 vision
//    tower over three 224x224 camera views.
//  The pages never print the formula; the scaled dot-product softmax above is
//  the computation nn.MultiheadAttention / FlashMHA perform.
//
// Inputs arrive either as fp64 arrays or as the packed [B,N,3,H,d] bf16 bit
// patterns that the qkv linear emits; bf16 is widened to fp64 exactly.
// Everything is accumulated and returned in fp64.  Work is spread over
// (b, h) pairs with std::thread; each (b, h) is computed by one thread in the
// order written above.

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstddef>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

double widen_bf16(uint16_t bits) {
  uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, sizeof(f));
  return static_cast<double>(f);
}

// One query row of one head.  qi points at the query's d channels; k and v
// point at key/value token 0, consecutive tokens `tok_stride` doubles apart,
// channels contiguous.  Writes d outputs to `oi`; if `probs` is non-null it
// also receives the N softmax weights of this row.  `s` is N doubles of
// workspace.
void one_row(const double* qi, const double* k, const double* v,
             std::ptrdiff_t tok_stride, int N, int d, double scale,
             double* oi, double* probs, double* s) {
  for (int j = 0; j < N; ++j) {
    const double* kj = k + j * tok_stride;
    double dot = 0.0;
    for (int c = 0; c < d; ++c) dot += qi[c] * kj[c];
    s[j] = scale * dot;
  }
  double m = s[0];
  for (int j = 1; j < N; ++j) m = std::max(m, s[j]);
  double l = 0.0;
  for (int j = 0; j < N; ++j) {
    s[j] = std::exp(s[j] - m);
    l += s[j];
  }
  for (int c = 0; c < d; ++c) {
    double acc = 0.0;
    for (int j = 0; j < N; ++j) acc += s[j] * v[j * tok_stride + c];
    oi[c] = acc / l;
  }
  if (probs != nullptr) {
    for (int j = 0; j < N; ++j) probs[j] = s[j] / l;
  }
}

// One (b, h) head: all N query rows.  Outputs have token stride `o_stride`;
// `probs`, if non-null, receives the N x N softmax matrix (row i = query i).
void one_head(const double* q, const double* k, const double* v,
              std::ptrdiff_t tok_stride, int N, int d, double scale,
              double* o, std::ptrdiff_t o_stride, double* probs) {
  std::vector<double> s(static_cast<size_t>(N));
  for (int i = 0; i < N; ++i) {
    one_row(q + i * tok_stride, k, v, tok_stride, N, d, scale, o + i * o_stride,
            probs ? probs + static_cast<size_t>(i) * N : nullptr, s.data());
  }
}

template <class F>
void parallel_for(long count, int nthreads, F&& body) {
  if (nthreads <= 0) {
    unsigned hc = std::thread::hardware_concurrency();
    nthreads = hc == 0 ? 1 : static_cast<int>(hc);
  }
  nthreads = static_cast<int>(std::min<long>(nthreads, std::max<long>(count, 1)));
  if (nthreads <= 1) {
    for (long t = 0; t < count; ++t) body(t);
    return;
  }
  std::atomic<long> next{0};
  std::vector<std::thread> pool;
  pool.reserve(static_cast<size_t>(nthreads));
  for (int w = 0; w < nthreads; ++w) {
    pool.emplace_back([&]() {
      for (long t = next.fetch_add(1); t < count; t = next.fetch_add(1)) body(t);
    });
  }
  for (auto& th : pool) th.join();
}

bool bad_shape(int B, int N, int H, int d) {
  return B < 0 || N < 0 || H < 0 || d <= 0;
}

}  // namespace

extern "C" {

// Number of worker threads a call with nthreads <= 0 uses.
int oracle_default_threads(void) {
  unsigned hc = std::thread::hardware_concurrency();
  return hc == 0 ? 1 : static_cast<int>(hc);
}

// q, k, v, o: contiguous fp64 [B, N, H, d].  Returns 0, or -1 on bad input.
int oracle_attn_f64(const double* q, const double* k, const double* v, double* o,
                    int B, int N, int H, int d, double scale, int nthreads) {
  if (bad_shape(B, N, H, d)) return -1;
  if (static_cast<long>(B) * N * H == 0) return 0;
  if (!q || !k || !v || !o) return -1;
  const std::ptrdiff_t tok = static_cast<std::ptrdiff_t>(H) * d;
  parallel_for(static_cast<long>(B) * H, nthreads, [&](long t) {
    const long b = t / H, h = t % H;
    const std::ptrdiff_t base = b * static_cast<std::ptrdiff_t>(N) * tok + h * d;
    one_head(q + base, k + base, v + base, tok, N, d, scale, o + base, tok, nullptr);
  });
  return 0;
}

// Softmax matrix: q, k contiguous fp64 [B, N, H, d]; p receives [B, H, N, N].
int oracle_attn_probs_f64(const double* q, const double* k, double* p,
                          int B, int N, int H, int d, double scale) {
  if (bad_shape(B, N, H, d)) return -1;
  if (static_cast<long>(B) * N * H == 0) return 0;
  if (!q || !k || !p) return -1;
  const std::ptrdiff_t tok = static_cast<std::ptrdiff_t>(H) * d;
  std::vector<double> scratch(static_cast<size_t>(N) * d);
  for (long b = 0; b < B; ++b) {
    for (long h = 0; h < H; ++h) {
      const std::ptrdiff_t base = b * static_cast<std::ptrdiff_t>(N) * tok + h * d;
      // v is irrelevant for the probabilities; reuse k as a stand-in.
      one_head(q + base, k + base, k + base, tok, N, d, scale, scratch.data(), d,
               p + (b * H + h) * static_cast<std::ptrdiff_t>(N) * N);
    }
  }
  return 0;
}

namespace {

// Widen the (b, h) slice of a packed [B,N,3,H,d] bf16 buffer into three
// contiguous N x d fp64 arrays.
void widen_head(const uint16_t* qkv, long b, long h, int N, int H, int d,
                std::vector<double>& q, std::vector<double>& k, std::vector<double>& v) {
  const std::ptrdiff_t tok = 3 * static_cast<std::ptrdiff_t>(H) * d;
  const std::ptrdiff_t hd = static_cast<std::ptrdiff_t>(H) * d;
  for (int n = 0; n < N; ++n) {
    const uint16_t* row = qkv + (b * N + n) * tok + h * d;
    for (int c = 0; c < d; ++c) {
      q[static_cast<size_t>(n) * d + c] = widen_bf16(row[c]);
      k[static_cast<size_t>(n) * d + c] = widen_bf16(row[hd + c]);
      v[static_cast<size_t>(n) * d + c] = widen_bf16(row[2 * hd + c]);
    }
  }
}

}  // namespace

// qkv: packed [B, N, 3, H, d] bf16 bit patterns; o: fp64 [B, N, H, d].
int oracle_attn_packed_bf16(const uint16_t* qkv, double* o, int B, int N, int H, int d,
                            double scale, int nthreads) {
  if (bad_shape(B, N, H, d)) return -1;
  if (static_cast<long>(B) * N * H == 0) return 0;
  if (!qkv || !o) return -1;
  const std::ptrdiff_t otok = static_cast<std::ptrdiff_t>(H) * d;
  parallel_for(static_cast<long>(B) * H, nthreads, [&](long t) {
    const long b = t / H, h = t % H;
    std::vector<double> q(static_cast<size_t>(N) * d), k(q.size()), v(q.size());
    widen_head(qkv, b, h, N, H, d, q, k, v);
    one_head(q.data(), k.data(), v.data(), d, N, d, scale,
             o + b * static_cast<std::ptrdiff_t>(N) * otok + h * d, otok, nullptr);
  });
  return 0;
}

// Selected output rows of a packed bf16 input: rows[3*r .. 3*r+2] = (b, h, n).
// out receives nrows x d fp64 values, each computed by the plain definition
// over the whole (b, h) head.
int oracle_attn_rows_packed_bf16(const uint16_t* qkv, int B, int N, int H, int d,
                                 double scale, const int64_t* rows, int nrows,
                                 double* out, int nthreads) {
  if (bad_shape(B, N, H, d) || nrows < 0) return -1;
  if (nrows == 0) return 0;
  if (!qkv || !rows || !out) return -1;
  for (int r = 0; r < nrows; ++r) {
    if (rows[3 * r] < 0 || rows[3 * r] >= B || rows[3 * r + 1] < 0 || rows[3 * r + 1] >= H ||
        rows[3 * r + 2] < 0 || rows[3 * r + 2] >= N)
      return -1;
  }
  parallel_for(nrows, nthreads, [&](long r) {
    const long b = rows[3 * r], h = rows[3 * r + 1], n = rows[3 * r + 2];
    std::vector<double> q(static_cast<size_t>(N) * d), k(q.size()), v(q.size());
    std::vector<double> s(static_cast<size_t>(N));
    widen_head(qkv, b, h, N, H, d, q, k, v);
    one_row(q.data() + n * d, k.data(), v.data(), d, N, d, scale, out + r * d, nullptr,
            s.data());
  });
  return 0;
}

// ---------------------------------------------------------------------------
// The two operations on either side of the attention core in a ViT block, in
// the same plain fp64 style (test infrastructure only, like the rest):
//
//   LayerNorm over the last dimension (width W) of every row m:
//     mu  = (1/W) sum_i x[m,i]
//     var = (1/W) sum_i (x[m,i] - mu)^2                (biased, as LayerNorm)
//     y[m,i] = (x[m,i] - mu) / sqrt(var + eps) * gamma[i] + beta[i]
//   "FluxVLA docs, inference acceleration", Triton fused kernels (norm
//   fusion: residual add + LayerNorm in one kernel); the ViT block applies it
//   before its qkv linear.
//
//   Linear layer with bias and optional residual (weight stored [N, K] as in
//   nn.Linear, i.e. the pages' weight(K,N) transposed):
//     y[m,n] = sum_k x[m,k] * w[n,k] + bias[n] + res[m,n]
//   same page, section 3, CUDA custom operators: cublasLt fused GEMM + bias
//   (+ residual), D = inp @ weight + bias (+ res); "Pi0 VLA deployment
//   tutorial", section 3.2: the block's qkv linear feeds the attention.
//
// bf16 inputs are widened exactly; bias and res may be null (treated as 0).

// LayerNorm of M rows of width W (bf16 x, gamma, beta) into fp64 y.
int oracle_layernorm_bf16(const uint16_t* x, const uint16_t* gamma, const uint16_t* beta,
                          double* y, int M, int W, double eps, int nthreads) {
  if (M < 0 || W <= 0 || !(eps >= 0.0)) return -1;
  parallel_for(static_cast<long>(M), nthreads, [&](long m) {
    const uint16_t* xm = x + m * static_cast<std::ptrdiff_t>(W);
    double sum = 0.0;
    for (int i = 0; i < W; ++i) sum += widen_bf16(xm[i]);
    const double mu = sum / W;
    double ss = 0.0;
    for (int i = 0; i < W; ++i) {
      const double dv = widen_bf16(xm[i]) - mu;
      ss += dv * dv;
    }
    const double var = ss / W;
    const double rstd = 1.0 / std::sqrt(var + eps);
    double* ym = y + m * static_cast<std::ptrdiff_t>(W);
    for (int i = 0; i < W; ++i)
      ym[i] = (widen_bf16(xm[i]) - mu) * rstd * widen_bf16(gamma[i]) + widen_bf16(beta[i]);
  });
  return 0;
}

// y[m,n] = sum_k x[m,k] w[n,k] + bias[n] + res[m,n]  (bf16 inputs, fp64 y).
int oracle_linear_bf16(const uint16_t* x, const uint16_t* w, const uint16_t* bias,
                       const uint16_t* res, double* y, int M, int K, int N, int nthreads) {
  if (M < 0 || K <= 0 || N <= 0) return -1;
  parallel_for(static_cast<long>(M), nthreads, [&](long m) {
    std::vector<double> xm(static_cast<size_t>(K));
    for (int k = 0; k < K; ++k) xm[k] = widen_bf16(x[m * static_cast<std::ptrdiff_t>(K) + k]);
    for (int n = 0; n < N; ++n) {
      const uint16_t* wn = w + n * static_cast<std::ptrdiff_t>(K);
      double acc = 0.0;
      for (int k = 0; k < K; ++k) acc += xm[k] * widen_bf16(wn[k]);
      if (bias != nullptr) acc += widen_bf16(bias[n]);
      if (res != nullptr) acc += widen_bf16(res[m * static_cast<std::ptrdiff_t>(N) + n]);
      y[m * static_cast<std::ptrdiff_t>(N) + n] = acc;
    }
  });
  return 0;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// The rest of a ViT encoder layer, same plain fp64 style:
//
//   Residual add + LayerNorm (one fused operator on the FluxVLA page, Triton
//   fused kernels: norm fusion).  The sum is the residual stream, which is
//   stored in bf16, and the LayerNorm reads that stored stream:
//     s[m,i] = bf16_rne(x[m,i] + r[m,i])       (returned as bf16 bits)
//     y[m,i] = LayerNorm(s)[m,i]               (as above, fp64)
//   The fusion must give what the two separate steps give, so s is rounded
//   exactly as an unfused add that stores bf16 would round it.
//
//   Linear layer + bias + GELU (same page, same section: matrix multiply with
//   bias and activation fused after the tiled product), the first MLP layer:
//     a[m,n] = sum_k x[m,k] * w[n,k] + bias[n]
//     y[m,n] = a/2 * (1 + tanh(sqrt(2/pi) * (a + 0.044715 a^3)))
//   The pages do not say which GELU; this is the tanh form of Hendrycks and
//   Gimpel's paper, the one SigLIP (the Pi0 vision encoder) uses.

namespace {

// Round-to-nearest-even of a finite double to bf16 (8 significant bits,
// 8 exponent bits), returned as bits.  From the format's definition: the
// value is scaled so that its quantum becomes 1, rounded to an integer with
// ties to even (the default floating-point rounding mode), and scaled back.
uint16_t round_bf16(double v) {
  if (v == 0.0) return std::signbit(v) ? 0x8000u : 0u;
  int e = 0;
  (void)std::frexp(v, &e);                     // |v| = f 2^e, f in [0.5, 1)
  const int q = std::max(e - 8, -133);         // quantum 2^q; subnormals share 2^-133
  const double r = std::ldexp(std::nearbyint(std::ldexp(v, -q)), q);
  if (std::fabs(r) >= std::ldexp(1.0, 128)) return std::signbit(v) ? 0xFF80u : 0x7F80u;
  const float f = static_cast<float>(r);       // exact: r has at most 8 significant bits
  uint32_t u;
  std::memcpy(&u, &f, sizeof(u));
  return static_cast<uint16_t>(u >> 16);
}

}  // namespace

extern "C" {

int oracle_round_bf16(const double* v, uint16_t* bits, long n) {
  for (long i = 0; i < n; ++i) {
    if (!std::isfinite(v[i])) return -1;
    bits[i] = round_bf16(v[i]);
  }
  return 0;
}

// s = bf16(x + r) (bits), y = LayerNorm(s) (fp64); M rows of width W.
int oracle_add_layernorm_bf16(const uint16_t* x, const uint16_t* r, const uint16_t* gamma,
                              const uint16_t* beta, uint16_t* s, double* y, int M, int W,
                              double eps, int nthreads) {
  if (M < 0 || W <= 0 || !(eps >= 0.0)) return -1;
  parallel_for(static_cast<long>(M), nthreads, [&](long m) {
    const std::ptrdiff_t off = m * static_cast<std::ptrdiff_t>(W);
    for (int i = 0; i < W; ++i)
      s[off + i] = round_bf16(widen_bf16(x[off + i]) + widen_bf16(r[off + i]));
  });
  return oracle_layernorm_bf16(s, gamma, beta, y, M, W, eps, nthreads);
}

// y[m,n] = gelu(sum_k x[m,k] w[n,k] + bias[n])  (bf16 inputs, fp64 y; bias may be null).
int oracle_linear_gelu_bf16(const uint16_t* x, const uint16_t* w, const uint16_t* bias,
                            double* y, int M, int K, int N, int nthreads) {
  const int rc = oracle_linear_bf16(x, w, bias, nullptr, y, M, K, N, nthreads);
  if (rc != 0) return rc;
  const double c = std::sqrt(2.0 / 3.14159265358979323846);
  const long n = static_cast<long>(M) * N;
  for (long i = 0; i < n; ++i) {
    const double a = y[i];
    y[i] = 0.5 * a * (1.0 + std::tanh(c * (a + 0.044715 * a * a * a)));
  }
  return 0;
}

}  // extern "C"
